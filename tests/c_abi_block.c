/*
 * A C caller of the library's C ABI (no Python): reads q, k and v ([B, T, H, D]
 * of `dtype`, raw element bytes, in that order) from argv[1], runs
 * scatter_sequence -> the Ulysses block (num_chunks from argv[3]) ->
 * gather_sequence on `world` virtual ranks (argv[4]) through include/usp.h, and
 * writes the [B, T, H, D] output (same dtype) to argv[2]. Sizes B T H D follow
 * in argv[5..8], the dtype ("bf16" or "fp32") in argv[9]. Exit status 0 on
 * success.
 * Used by tests/test_gpu_c_abi.py, which compares the output with the oracle.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "usp.h"

#define CHECK_USP(call)                                                                 \
  do {                                                                                  \
    int rc_ = (call);                                                                   \
    if (rc_ != USP_OK) {                                                                \
      fprintf(stderr, "%s failed (%d): %s\n", #call, rc_, usp_last_error_message());  \
      return 1;                                                                         \
    }                                                                                   \
  } while (0)
#define CHECK_CUDA(call)                                                              \
  do {                                                                                \
    cudaError_t e_ = (call);                                                          \
    if (e_ != cudaSuccess) {                                                          \
      fprintf(stderr, "%s failed: %s\n", #call, cudaGetErrorString(e_));              \
      return 1;                                                                       \
    }                                                                                 \
  } while (0)

int main(int argc, char** argv) {
  if (argc != 10) {
    fprintf(stderr, "usage: %s in.bin out.bin num_chunks world B T H D bf16|fp32\n", argv[0]);
    return 2;
  }
  const int bf16 = strcmp(argv[9], "bf16") == 0;
  const size_t elem = bf16 ? 2 : 4;
  const int num_chunks = atoi(argv[3]), world = atoi(argv[4]);
  const int64_t B = atoll(argv[5]), T = atoll(argv[6]);
  const int32_t H = atoi(argv[7]), D = atoi(argv[8]);
  const size_t n = (size_t)(B * T * H * D), bytes = n * elem;

  char* host = (char*)malloc(3 * bytes);
  FILE* f = fopen(argv[1], "rb");
  if (!host || !f || fread(host, 1, 3 * bytes, f) != 3 * bytes) {
    fprintf(stderr, "cannot read %s\n", argv[1]);
    return 1;
  }
  fclose(f);

  usp_plan* plan = NULL;
  CHECK_USP(usp_plan_create(&plan, B, T, H, D, world, bf16 ? USP_BF16 : USP_FP32, 0));
  int64_t tok_len[USP_MAX_WORLD];
  CHECK_USP(usp_plan_query(plan, NULL, tok_len, NULL, NULL));

  cudaStream_t s;
  CHECK_CUDA(cudaStreamCreate(&s));
  void* full[3];
  void* shards[3][USP_MAX_WORLD];
  void* out[USP_MAX_WORLD];
  for (int t = 0; t < 3; ++t) {
    CHECK_CUDA(cudaMalloc(&full[t], bytes));
    CHECK_CUDA(cudaMemcpy(full[t], host + t * bytes, bytes, cudaMemcpyHostToDevice));
    for (int r = 0; r < world; ++r)
      CHECK_CUDA(cudaMalloc(&shards[t][r], (size_t)(B * tok_len[r] * H * D) * elem));
    CHECK_USP(usp_scatter_sequence(plan, full[t], shards[t], 0, 0, s));
  }
  for (int r = 0; r < world; ++r) CHECK_CUDA(cudaMalloc(&out[r], (size_t)(B * tok_len[r] * H * D) * elem));

  size_t ws_bytes = 0;
  CHECK_USP(usp_ulysses_attention_workspace_size(plan, num_chunks, &ws_bytes));
  void* ws = NULL;
  CHECK_CUDA(cudaMalloc(&ws, ws_bytes));
  CHECK_USP(usp_ulysses_attention(plan, (const void* const*)shards[0], (const void* const*)shards[1],
                                  (const void* const*)shards[2], out, 0.0f, num_chunks, ws, ws_bytes, s));
  CHECK_USP(usp_gather_sequence(plan, (const void* const*)out, full[0], 0, 0, s));
  CHECK_CUDA(cudaStreamSynchronize(s));
  uint32_t code = 0;
  CHECK_USP(usp_device_status(&code, 1));

  CHECK_CUDA(cudaMemcpy(host, full[0], bytes, cudaMemcpyDeviceToHost));
  f = fopen(argv[2], "wb");
  if (!f || fwrite(host, 1, bytes, f) != bytes) {
    fprintf(stderr, "cannot write %s\n", argv[2]);
    return 1;
  }
  fclose(f);

  for (int t = 0; t < 3; ++t) {
    cudaFree(full[t]);
    for (int r = 0; r < world; ++r) cudaFree(shards[t][r]);
  }
  for (int r = 0; r < world; ++r) cudaFree(out[r]);
  cudaFree(ws);
  cudaStreamDestroy(s);
  CHECK_USP(usp_plan_destroy(plan));
  free(host);
  printf("ok version %d\n", usp_version());
  return 0;
}
