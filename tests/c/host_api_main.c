/*
 * A plain C caller of the streaming_top C ABI: reads an indexer problem from
 * a binary file, runs si_indexer_topk_host (host buffers in, host buffers
 * out) and writes the results to a binary file.  Built by the test suite with
 * gcc against include/streaming_top.h and libstreaming_top.so.
 *
 * Input file:  int32 B, R, T, H_I, D, m, k, row0, query_chunk; then q
 *              [B,R,H_I,D] bf16 bits (uint16), kc [B,T,D] bf16 bits, w
 *              [B,R,H_I] fp32.
 * Output file: int32 status; then out_idx [B,R,k] int32, out_score [B,R,k]
 *              fp32.
 * Usage: host_api_main IN OUT.  The host buffers are plain malloc memory
 * (pageable), so the library's copies run synchronously; the results are the
 * same as with page-locked buffers.
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "streaming_top.h"

static void* read_exact(FILE* f, size_t bytes) {
  void* p = malloc(bytes ? bytes : 1);
  if (!p || fread(p, 1, bytes, f) != bytes) {
    fprintf(stderr, "short read (%zu bytes)\n", bytes);
    exit(2);
  }
  return p;
}

int main(int argc, char** argv) {
  if (argc < 3) {
    fprintf(stderr, "usage: %s IN OUT\n", argv[0]);
    return 2;
  }
  FILE* f = fopen(argv[1], "rb");
  if (!f) {
    perror(argv[1]);
    return 2;
  }
  int32_t hdr[9];
  if (fread(hdr, sizeof hdr, 1, f) != 1) {
    fprintf(stderr, "short header\n");
    return 2;
  }
  const int B = hdr[0], R = hdr[1], T = hdr[2], H = hdr[3], D = hdr[4], m = hdr[5], k = hdr[6];
  const int row0 = hdr[7], chunk = hdr[8];
  const size_t nq = (size_t)B * R * H * D, nk = (size_t)B * T * D, nw = (size_t)B * R * H, no = (size_t)B * R * k;
  void* q = read_exact(f, nq * 2);
  void* kc = read_exact(f, nk * 2);
  float* w = (float*)read_exact(f, nw * 4);
  fclose(f);
  int32_t* idx = (int32_t*)malloc(no * 4);
  float* score = (float*)malloc(no * 4);
  si_options opt;
  memset(&opt, 0, sizeof opt);
  opt.dtype = SI_DTYPE_BF16;
  opt.query_chunk = chunk;
  const si_status st = si_indexer_topk_host(q, kc, w, B, row0, R, T, H, D, m, k, idx, score, NULL, &opt);
  if (st != SI_OK) fprintf(stderr, "si_indexer_topk_host: %s: %s\n", si_status_string(st), si_last_error());
  FILE* o = fopen(argv[2], "wb");
  if (!o) {
    perror(argv[2]);
    return 2;
  }
  const int32_t s32 = (int32_t)st;
  fwrite(&s32, 4, 1, o);
  fwrite(idx, 4, no, o);
  fwrite(score, 4, no, o);
  fclose(o);
  free(q);
  free(kc);
  free(w);
  free(idx);
  free(score);
  return st == SI_OK ? 0 : 1;
}
