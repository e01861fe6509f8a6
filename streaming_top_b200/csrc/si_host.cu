// si_indexer_topk_host: the streaming indexer top-k on host buffers.
//
// The pages stream the queries through the indexer in chunks so that only
// one chunk is resident at a time (StreamIndex abstract: the memory bound at
// a million tokens).  This entry point does the same from host memory: the
// keys are copied once, then the query rows go through the device in chunks
// of `query_chunk` rows through two slots, so that the copy of chunk c+1 in,
// the scoring of chunk c and the copy of chunk c-1 out overlap:
//
//   copy-in stream    H2D q/w(c)   H2D q/w(c+1)   H2D q/w(c+2) ...
//   caller's stream                score(c)       score(c+1)   ...
//   copy-out stream                               D2H out(c)   ...
//
// ordered by events: slot s = c % 2 takes chunk c's inputs only after
// chunk c-2's scoring has read them, and chunk c's results only after chunk
// c-2's have been copied out.  Every copy is a plain cudaMemcpyAsync (one
// per sequence of a chunk), never a batched-copy call.  The call returns
// when the results are in the host buffers.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "si_internal.h"

namespace si {
namespace {

constexpr int kDefaultHostChunk = 4096;
constexpr int kSlots = 2;

struct HostPlan {
  int R;             // rows per chunk
  size_t q_row;      // bytes of one query row of q (H_I * D * element size)
  size_t kc_row;     // bytes of one key row as given (bf16 / e4m3 / MXFP4 codes)
  size_t off_kc, off_kc_scale, off_mx_scale, off_kdec;
  size_t off_slot[kSlots];
  size_t slot_q, slot_w, slot_qs, slot_idx, slot_sc;  // offsets within a slot
  size_t total;
};

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

HostPlan plan(int B, int rows, int T, int H, int D, int k, bool with_score, const si_options& o) {
  HostPlan p;
  const bool fp8 = o.dtype == SI_DTYPE_FP8_E4M3, mx = o.dtype == SI_DTYPE_MXFP4_KEYS;
  p.R = std::min(o.query_chunk > 0 ? o.query_chunk : kDefaultHostChunk, rows);
  p.q_row = static_cast<size_t>(H) * D * (fp8 ? 1 : 2);
  p.kc_row = mx ? static_cast<size_t>(D) / 2 : static_cast<size_t>(D) * (fp8 ? 1 : 2);
  size_t cur = 0;
  p.off_kc = cur;
  cur = up256(cur + static_cast<size_t>(B) * T * p.kc_row);
  p.off_kc_scale = cur;
  if (fp8) cur = up256(cur + static_cast<size_t>(B) * T * 4);
  p.off_mx_scale = cur;
  if (mx) cur = up256(cur + static_cast<size_t>(B) * T * (D / 32));
  p.off_kdec = cur;
  if (mx) cur = up256(cur + static_cast<size_t>(B) * T * D * 2);
  const size_t br = static_cast<size_t>(B) * p.R;
  size_t sc = 0;
  p.slot_q = sc;
  sc = up256(sc + br * p.q_row);
  p.slot_w = sc;
  sc = up256(sc + br * H * 4);
  p.slot_qs = sc;
  if (fp8) sc = up256(sc + br * H * 4);
  p.slot_idx = sc;
  sc = up256(sc + br * k * 4);
  p.slot_sc = sc;
  if (with_score) sc = up256(sc + br * k * 4);
  for (int s = 0; s < kSlots; ++s) {
    p.off_slot[s] = cur;
    cur += sc;
  }
  p.total = cur + 256;  // alignment slack of the base
  return p;
}

si_status check_host_args(const void* q, const void* kc, const float* w, int B, int row0, int R, int T,
                          int H, int D, int m, int k, const int32_t* out_idx, const si_options& o) {
  if (!q || !kc || !w || !out_idx)
    return fail(SI_ERR_INVALID_ARGUMENT, "q, kc, w and out_idx must be non-null host pointers");
  if (B < 1 || R < 1 || T < 1 || H < 1 || D < 1 || m < 1 || k < 1)
    return fail(SI_ERR_INVALID_ARGUMENT, "B, R, T, H_I, D, m, k must be >= 1 (got %d %d %d %d %d %d %d)", B, R,
                T, H, D, m, k);
  if (row0 < 0) return fail(SI_ERR_INVALID_ARGUMENT, "row0 must be >= 0 (got %d)", row0);
  if (static_cast<long long>(row0) + R > 0x7FFFFFFFll)
    return fail(SI_ERR_UNSUPPORTED, "row0 + rows must fit in 31 bits");
  if (o.dtype != SI_DTYPE_BF16 && o.dtype != SI_DTYPE_FP8_E4M3 && o.dtype != SI_DTYPE_MXFP4_KEYS)
    return fail(SI_ERR_INVALID_ARGUMENT, "unknown dtype %d", static_cast<int>(o.dtype));
  if (o.dtype == SI_DTYPE_FP8_E4M3 && (!o.q_scale || !o.kc_scale))
    return fail(SI_ERR_INVALID_ARGUMENT, "fp8 inputs need q_scale and kc_scale");
  if (o.dtype == SI_DTYPE_MXFP4_KEYS && !o.kc_mx_scale)
    return fail(SI_ERR_INVALID_ARGUMENT, "MXFP4 keys need kc_mx_scale");
  if (o.query_chunk < 0 || (o.query_chunk % 4) != 0)
    return fail(SI_ERR_INVALID_ARGUMENT, "query_chunk must be 0 or a positive multiple of 4 (got %d)",
                o.query_chunk);
  if (D != 128 || H != 64)
    return fail(SI_ERR_UNSUPPORTED, "streaming path implements D=128, H_I=64 (got D=%d, H_I=%d)", D, H);
  if (k > 2048) return fail(SI_ERR_UNSUPPORTED, "k <= 2048 (got %d)", k);
  return SI_OK;
}

// Copies `height` rows of `width` bytes (one per sequence) between pitched
// layouts, one cudaMemcpyAsync per row (the pitches of a long sequence can
// exceed what a 2D copy accepts).
si_status copy2d(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width, size_t height,
                 cudaMemcpyKind kind, cudaStream_t s, const char* what) {
  for (size_t r = 0; r < height; ++r) {
    const cudaError_t e = cudaMemcpyAsync(static_cast<uint8_t*>(dst) + r * dpitch,
                                          static_cast<const uint8_t*>(src) + r * spitch, width, kind, s);
    if (e != cudaSuccess) return cuda_fail(e, what);
  }
  return SI_OK;
}

}  // namespace
}  // namespace si

using namespace si;

extern "C" {

size_t si_indexer_topk_host_workspace_size(int B, int R, int T, int H_I, int D, int k, int with_score,
                                           const si_options* opt) {
  if (B < 1 || R < 1 || T < 1 || H_I < 1 || D < 1 || k < 1) return 0;
  si_options o;
  std::memset(&o, 0, sizeof o);
  if (opt) o = *opt;
  if (o.query_chunk < 0) return 0;
  return plan(B, R, T, H_I, D, k, with_score != 0, o).total;
}

si_status si_indexer_topk_host(const void* q, const void* kc, const float* w, int B, int row0, int R, int T,
                               int H_I, int D, int m, int k, int32_t* out_idx, float* out_score,
                               void* stream, const si_options* opt) {
  si_options o;
  std::memset(&o, 0, sizeof o);
  if (opt) o = *opt;
  si_status st = check_host_args(q, kc, w, B, row0, R, T, H_I, D, m, k, out_idx, o);
  if (st != SI_OK) return st;
  const bool fp8 = o.dtype == SI_DTYPE_FP8_E4M3, mx = o.dtype == SI_DTYPE_MXFP4_KEYS;
  const HostPlan P = plan(B, R, T, H_I, D, k, out_score != nullptr, o);
  if (o.workspace && o.workspace_bytes < P.total)
    return fail(SI_ERR_INVALID_ARGUMENT, "workspace of %zu bytes < %zu needed", o.workspace_bytes, P.total);

  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  void* raw = nullptr;
  if (!o.workspace) {
    st = scratch_alloc(&raw, P.total, cs, "the host-buffer call's device buffers");
    if (st != SI_OK) return st;
  }
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(o.workspace ? o.workspace : raw) + 255) & ~static_cast<uintptr_t>(255));

  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_ready = nullptr, ev_in[kSlots] = {}, ev_comp[kSlots] = {}, ev_out[kSlots] = {},
              ev_in_end = nullptr, ev_out_end = nullptr;
  cudaError_t e = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking);
  cudaEvent_t* all_ev[] = {&ev_ready, &ev_in[0], &ev_in[1], &ev_comp[0], &ev_comp[1],
                           &ev_out[0], &ev_out[1], &ev_in_end, &ev_out_end};
  for (cudaEvent_t* ev : all_ev)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  if (e != cudaSuccess) st = cuda_fail(e, "creating the copy streams and events");

  // the copy-in stream starts after the buffers exist (stream-ordered allocation on cs)
  if (st == SI_OK) {
    e = cudaEventRecord(ev_ready, cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev_ready, 0);
    if (e != cudaSuccess) st = cuda_fail(e, "ordering the copy stream");
  }
  // keys (and their scales) once
  const size_t kc_bytes = static_cast<size_t>(B) * T * P.kc_row;
  if (st == SI_OK) {
    e = cudaMemcpyAsync(base + P.off_kc, kc, kc_bytes, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess && fp8)
      e = cudaMemcpyAsync(base + P.off_kc_scale, o.kc_scale, static_cast<size_t>(B) * T * 4,
                          cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess && mx)
      e = cudaMemcpyAsync(base + P.off_mx_scale, o.kc_mx_scale, static_cast<size_t>(B) * T * (D / 32),
                          cudaMemcpyHostToDevice, s_in);
    if (e != cudaSuccess) st = cuda_fail(e, "copying the keys to the device");
  }
  // the options every chunk runs with: device scales, the decoded keys for MXFP4
  si_options oc = o;
  oc.workspace = nullptr;
  oc.workspace_bytes = 0;
  oc.query_chunk = 0;
  oc.q_scale = nullptr;
  oc.kc_scale = fp8 ? reinterpret_cast<const float*>(base + P.off_kc_scale) : nullptr;
  oc.kc_mx_scale = nullptr;
  const void* kc_dev = base + P.off_kc;
  if (mx) {
    oc.dtype = SI_DTYPE_BF16;
    kc_dev = base + P.off_kdec;
  }

  const int n_chunks = (R + P.R - 1) / P.R;
  bool keys_ready = false;
  for (int c = 0; c < n_chunks && st == SI_OK; ++c) {
    const int s = c % kSlots;
    const int r0 = c * P.R, n = std::min(P.R, R - r0);
    uint8_t* slot = base + P.off_slot[s];
    // inputs: wait until chunk c-2's scoring has read this slot
    if (c >= kSlots) {
      e = cudaStreamWaitEvent(s_in, ev_comp[s], 0);
      if (e != cudaSuccess) {
        st = cuda_fail(e, "ordering the copy-in stream");
        break;
      }
    }
    st = copy2d(slot + P.slot_q, n * P.q_row, static_cast<const uint8_t*>(q) + r0 * P.q_row, R * P.q_row,
                n * P.q_row, B, cudaMemcpyHostToDevice, s_in, "copying q rows in");
    if (st == SI_OK)
      st = copy2d(slot + P.slot_w, static_cast<size_t>(n) * H_I * 4, w + static_cast<size_t>(r0) * H_I,
                  static_cast<size_t>(R) * H_I * 4, static_cast<size_t>(n) * H_I * 4, B, cudaMemcpyHostToDevice,
                  s_in, "copying w rows in");
    if (st == SI_OK && fp8)
      st = copy2d(slot + P.slot_qs, static_cast<size_t>(n) * H_I * 4, o.q_scale + static_cast<size_t>(r0) * H_I,
                  static_cast<size_t>(R) * H_I * 4, static_cast<size_t>(n) * H_I * 4, B, cudaMemcpyHostToDevice,
                  s_in, "copying q scales in");
    if (st != SI_OK) break;
    e = cudaEventRecord(ev_in[s], s_in);
    // scoring: after the inputs landed and chunk c-2's results left the slot
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ev_in[s], 0);
    if (e == cudaSuccess && c >= kSlots) e = cudaStreamWaitEvent(cs, ev_out[s], 0);
    if (e != cudaSuccess) {
      st = cuda_fail(e, "ordering the compute stream");
      break;
    }
    if (mx && !keys_ready) {
      // the keys arrived with the first chunk's inputs: decode them once
      st = launch_mxfp4_to_bf16(base + P.off_kc, base + P.off_mx_scale, static_cast<long long>(B) * T, D,
                                base + P.off_kdec, cs);
      if (st != SI_OK) break;
    }
    keys_ready = true;
    oc.q_scale = fp8 ? reinterpret_cast<const float*>(slot + P.slot_qs) : nullptr;
    int32_t* idx_d = reinterpret_cast<int32_t*>(slot + P.slot_idx);
    float* sc_d = out_score ? reinterpret_cast<float*>(slot + P.slot_sc) : nullptr;
    st = stream_topk_rows(slot + P.slot_q, kc_dev, reinterpret_cast<const float*>(slot + P.slot_w), B, row0 + r0,
                          n, T, H_I, D, m, k, idx_d, sc_d, cs, &oc);
    if (st != SI_OK) break;
    e = cudaEventRecord(ev_comp[s], cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_comp[s], 0);
    if (e != cudaSuccess) {
      st = cuda_fail(e, "ordering the copy-out stream");
      break;
    }
    const size_t ob = static_cast<size_t>(n) * k * 4;
    st = copy2d(out_idx + static_cast<size_t>(r0) * k, static_cast<size_t>(R) * k * 4, idx_d, ob, ob, B,
                cudaMemcpyDeviceToHost, s_out, "copying indices out");
    if (st == SI_OK && out_score)
      st = copy2d(out_score + static_cast<size_t>(r0) * k, static_cast<size_t>(R) * k * 4, sc_d, ob, ob, B,
                  cudaMemcpyDeviceToHost, s_out, "copying scores out");
    if (st != SI_OK) break;
    e = cudaEventRecord(ev_out[s], s_out);
    if (e != cudaSuccess) st = cuda_fail(e, "recording the copy-out event");
  }

  // whatever happened: every copy and kernel is done before the buffers go
  if (s_in && s_out && ev_in_end && ev_out_end) {
    cudaEventRecord(ev_in_end, s_in);
    cudaEventRecord(ev_out_end, s_out);
    cudaStreamWaitEvent(cs, ev_in_end, 0);
    cudaStreamWaitEvent(cs, ev_out_end, 0);
  }
  if (raw) {
    e = cudaFreeAsync(raw, cs);
    if (e != cudaSuccess && st == SI_OK) st = cuda_fail(e, "cudaFreeAsync");
  }
  e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess && st == SI_OK) st = cuda_fail(e, "cudaStreamSynchronize");
  if (s_in) cudaStreamSynchronize(s_in);
  if (s_out) cudaStreamSynchronize(s_out);
  for (cudaEvent_t* ev : all_ev)
    if (*ev) cudaEventDestroy(*ev);
  if (s_in) cudaStreamDestroy(s_in);
  if (s_out) cudaStreamDestroy(s_out);
  if (st != SI_OK) return st;

  // the results are in host memory: report a bounded wait that ran out
  if (o.device_status) {
    int32_t h[2] = {0, 0};
    e = cudaMemcpy(h, o.device_status, sizeof h, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the call's status word");
    if (h[0] != 0) return fail(static_cast<si_status>(h[0]), "a kernel's bounded wait ran out (site %d)", h[1]);
    return SI_OK;
  }
  return si_device_status(stream);
}

}  // extern "C"
