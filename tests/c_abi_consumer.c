/* A plain C11 consumer of the C ABI (include/cmr.h), used by
 * tests/test_c_consumer.py.
 *   ./consumer host    -- version, status strings and host-side argument
 *                         checks; never touches a GPU
 *   ./consumer device  -- the planes of one 80-token prompt with <image> at
 *                         index 6, in cudaMalloc'd buffers; prints "p T H W"
 *                         lines and "start amount" for the test to compare,
 *                         then "frames same" if the multi-frame entry point
 *                         without a workspace gives the same planes, and
 *                         "host batch same" if the whole path on a batch in
 *                         cudaHostAlloc'd memory gives the device path's
 *                         planes, state and rotated Q/K bytes */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "cmr.h"

#define CHECK(cond)                                             \
  do {                                                          \
    if (!(cond)) {                                              \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      return 1;                                                 \
    }                                                           \
  } while (0)

static int host_checks(void) {
  CHECK(cmr_version() >= 20000);
  CHECK(strcmp(cmr_status_string(CMR_OK), "CMR_OK") == 0);
  const int32_t sections[3] = {11, 11, 10};
  const int32_t bad_sections[3] = {12, 11, 10};
  /* nothing to do */
  CHECK(cmr_rotate_qk(NULL, NULL, NULL, 0, 1, 8, 2, 256, 1e7, sections, 64, NULL, NULL) == CMR_OK);
  CHECK(cmr_positions(NULL, NULL, 0, 0, 248078, NULL, NULL, NULL, NULL, NULL) == CMR_OK);
  /* rejected before any CUDA call */
  void* fake = (void*)(uintptr_t)0x10000;
  CHECK(cmr_rotate_qk(fake, fake, fake, 10, 1, 8, 2, 256, 1e7, bad_sections, 64, NULL, NULL) == CMR_EINVAL);
  CHECK(strlen(cmr_last_error_message()) > 0);
  CHECK(cmr_rotate_qk(fake, fake, fake, 10, 1, 8, 2, 256, -1.0, sections, 64, NULL, NULL) == CMR_EINVAL);
  CHECK(cmr_rotate_qk(fake, fake, fake, 10, 1, 8, 2, 250, 1e7, sections, 64, NULL, NULL) == CMR_EINVAL);
  CHECK(cmr_positions(fake, NULL, 1, 10, 248078, fake, fake, fake, NULL, NULL) == CMR_EINVAL);
  CHECK(cmr_positions_chunk(fake, fake, 1, 10, 248078, 7, NULL, NULL, NULL, fake, fake, fake,
                            NULL, NULL) == CMR_EINVAL);
  CHECK(cmr_copy_rotated_dims(fake, fake, 4, 64, 128, 0, NULL) == CMR_EINVAL);
  /* which kernel a shape runs: pure host logic */
  CHECK(strcmp(cmr_rotate_qk_kernel(262144, 6, 8, 2, 256, 64), "rotate_qk_staged_kernel") == 0);
  CHECK(strcmp(cmr_rotate_qk_kernel(1024, 6, 8, 2, 256, 64), "rotate_qk_kernel") == 0);
  CHECK(strcmp(cmr_rotate_qk_cache_kernel(262144, 6, 8, 2, 256, 64),
               "rotate_qk_cache_staged_kernel") == 0);
  CHECK(cmr_rotate_qk_kernel(0, 6, 8, 2, 256, 64) == NULL);
  CHECK(strcmp(cmr_last_rotate_kernel(), "") == 0); /* nothing launched yet */
  /* the one-call path: nothing to do, and its rotate arguments are checked */
  CHECK(cmr_positions_rotate_qk(NULL, NULL, 0, 0, 248078, NULL, NULL, NULL, NULL, NULL, 1, 8, 2,
                                256, 1e7, sections, 64, NULL, NULL) == CMR_OK);
  CHECK(cmr_positions_rotate_qk(NULL, NULL, 0, 0, 248078, NULL, NULL, NULL, NULL, NULL, 1, 8, 2,
                                256, 1e7, bad_sections, 64, NULL, NULL) == CMR_EINVAL);
  /* several frames per prompt: the workspace size and the host checks */
  CHECK(cmr_positions_frames_workspace_bytes(32, 32 * 8192) == 16u * 32 * 2);
  CHECK(cmr_positions_rotate_qk_host(NULL, NULL, 0, 0, 248078, NULL, NULL, NULL, NULL, NULL, 1,
                                     8, 2, 256, 1e7, sections, 64, NULL, NULL) == CMR_OK);
  CHECK(cmr_positions_frames(fake, fake, 1, 10, 248078, 0, fake, fake, fake, fake, 1 << 20, NULL,
                             NULL) == CMR_EINVAL);
  CHECK(cmr_positions_frames_noalloc(fake, fake, 16385, 16385, 248078, 8, fake, fake, fake, NULL,
                                     NULL) == CMR_EINVAL);
  printf("host ok\n");
  return 0;
}

/* Just the CUDA runtime calls this program needs, declared here so that the
 * consumer compiles as plain C with gcc; linked from libcudart. */
typedef int cuda_err;
extern cuda_err cudaMalloc(void** p, size_t bytes);
extern cuda_err cudaFree(void* p);
extern cuda_err cudaMemcpy(void* dst, const void* src, size_t bytes, int kind);
extern cuda_err cudaDeviceSynchronize(void);
extern cuda_err cudaHostAlloc(void** p, size_t bytes, unsigned int flags);
extern cuda_err cudaFreeHost(void* p);
#define HOST_ALLOC_MAPPED 2u /* cudaHostAllocMapped */

static int device_run(void) {
  enum { N = 80, O = 6 };
  int32_t ids[N], cu[2] = {0, N};
  for (int p = 0; p < N; ++p) ids[p] = 1000 + p; /* text */
  ids[O] = 248078;                              /* <image> */
  for (int k = 0; k < 64; ++k) ids[O + 1 + k] = 248094 + k;
  ids[O + 65] = 248079;                         /* </image> */
  ids[O + 66] = 198;                            /* "\n" */
  int32_t *d_ids, *d_cu, *d_pos, *d_start, *d_amount;
  CHECK(cudaMalloc((void**)&d_ids, sizeof ids) == 0);
  CHECK(cudaMalloc((void**)&d_cu, sizeof cu) == 0);
  CHECK(cudaMalloc((void**)&d_pos, 3 * N * sizeof(int32_t)) == 0);
  CHECK(cudaMalloc((void**)&d_start, sizeof(int32_t)) == 0);
  CHECK(cudaMalloc((void**)&d_amount, sizeof(int32_t)) == 0);
  CHECK(cudaMemcpy(d_ids, ids, sizeof ids, 1) == 0);
  CHECK(cudaMemcpy(d_cu, cu, sizeof cu, 1) == 0);
  cmr_status s = cmr_positions(d_ids, d_cu, 1, N, 248078, d_pos, d_start, d_amount, NULL, NULL);
  if (s != CMR_OK) {
    fprintf(stderr, "cmr_positions: %s\n", cmr_last_error_message());
    return 1;
  }
  CHECK(cudaDeviceSynchronize() == 0);
  int32_t pos[3 * N], start, amount;
  CHECK(cudaMemcpy(pos, d_pos, sizeof pos, 2) == 0);
  CHECK(cudaMemcpy(&start, d_start, sizeof start, 2) == 0);
  CHECK(cudaMemcpy(&amount, d_amount, sizeof amount, 2) == 0);
  for (int p = 0; p < N; ++p) printf("%d %d %d %d\n", p, pos[p], pos[N + p], pos[2 * N + p]);
  printf("%d %d\n", start, amount);
  /* one frame at grid side 8 through the entry point that allocates nothing */
  int32_t* d_pos2;
  CHECK(cudaMalloc((void**)&d_pos2, 3 * N * sizeof(int32_t)) == 0);
  s = cmr_positions_frames_noalloc(d_ids, d_cu, 1, N, 248078, 8, d_pos2, d_start, d_amount, NULL,
                                   NULL);
  if (s != CMR_OK) {
    fprintf(stderr, "cmr_positions_frames_noalloc: %s\n", cmr_last_error_message());
    return 1;
  }
  CHECK(cudaDeviceSynchronize() == 0);
  int32_t pos2[3 * N];
  CHECK(cudaMemcpy(pos2, d_pos2, sizeof pos2, 2) == 0);
  if (memcmp(pos, pos2, sizeof pos) == 0) printf("frames same\n");
  /* the whole path on a batch in mapped page-locked host memory, against the
     same call on device copies */
  {
    enum { HQ = 8, HK = 2, D = 256 };
    const int32_t sections[3] = {11, 11, 10};
    const size_t qn = (size_t)N * HQ * D, kn = (size_t)N * HK * D;
    int32_t *h_ids, *h_cu, *h_pos, *h_start, *h_amount;
    uint16_t *h_q, *h_k, *d_q, *d_k;
    CHECK(cudaHostAlloc((void**)&h_ids, sizeof ids, HOST_ALLOC_MAPPED) == 0);
    CHECK(cudaHostAlloc((void**)&h_cu, sizeof cu, HOST_ALLOC_MAPPED) == 0);
    CHECK(cudaHostAlloc((void**)&h_pos, 3 * N * sizeof(int32_t), HOST_ALLOC_MAPPED) == 0);
    CHECK(cudaHostAlloc((void**)&h_start, sizeof(int32_t), HOST_ALLOC_MAPPED) == 0);
    CHECK(cudaHostAlloc((void**)&h_amount, sizeof(int32_t), HOST_ALLOC_MAPPED) == 0);
    CHECK(cudaHostAlloc((void**)&h_q, qn * 2, HOST_ALLOC_MAPPED) == 0);
    CHECK(cudaHostAlloc((void**)&h_k, kn * 2, HOST_ALLOC_MAPPED) == 0);
    CHECK(cudaMalloc((void**)&d_q, qn * 2) == 0);
    CHECK(cudaMalloc((void**)&d_k, kn * 2) == 0);
    memcpy(h_ids, ids, sizeof ids);
    memcpy(h_cu, cu, sizeof cu);
    /* bf16 values of magnitude 0.5 .. 2 with both signs, from a fixed LCG */
    uint32_t r = 12345u;
    for (size_t i = 0; i < qn; ++i) { r = r * 1664525u + 1013904223u; h_q[i] = (uint16_t)(0x3f00u + (r >> 25) + ((r >> 24) & 1u) * 0x8000u); }
    for (size_t i = 0; i < kn; ++i) { r = r * 1664525u + 1013904223u; h_k[i] = (uint16_t)(0x3f00u + (r >> 25) + ((r >> 24) & 1u) * 0x8000u); }
    CHECK(cudaMemcpy(d_q, h_q, qn * 2, 1) == 0);
    CHECK(cudaMemcpy(d_k, h_k, kn * 2, 1) == 0);
    s = cmr_positions_rotate_qk(d_ids, d_cu, 1, N, 248078, d_pos, d_start, d_amount, d_q, d_k, 1,
                                HQ, HK, D, 1e7, sections, 64, NULL, NULL);
    if (s != CMR_OK) {
      fprintf(stderr, "cmr_positions_rotate_qk: %s\n", cmr_last_error_message());
      return 1;
    }
    s = cmr_positions_rotate_qk_host(h_ids, h_cu, 1, N, 248078, h_pos, h_start, h_amount, h_q,
                                     h_k, 1, HQ, HK, D, 1e7, sections, 64, NULL, NULL);
    if (s != CMR_OK) {
      fprintf(stderr, "cmr_positions_rotate_qk_host: %s\n", cmr_last_error_message());
      return 1;
    }
    CHECK(cudaDeviceSynchronize() == 0);
    uint16_t* q_dev = malloc(qn * 2);
    uint16_t* k_dev = malloc(kn * 2);
    CHECK(q_dev && k_dev);
    CHECK(cudaMemcpy(q_dev, d_q, qn * 2, 2) == 0);
    CHECK(cudaMemcpy(k_dev, d_k, kn * 2, 2) == 0);
    CHECK(cudaMemcpy(pos2, d_pos, sizeof pos2, 2) == 0);
    if (memcmp(h_pos, pos2, sizeof pos2) == 0 && memcmp(h_pos, pos, sizeof pos) == 0 &&
        *h_start == start && *h_amount == amount && memcmp(h_q, q_dev, qn * 2) == 0 &&
        memcmp(h_k, k_dev, kn * 2) == 0)
      printf("host batch same\n");
    free(q_dev);
    free(k_dev);
    cudaFreeHost(h_ids);
    cudaFreeHost(h_cu);
    cudaFreeHost(h_pos);
    cudaFreeHost(h_start);
    cudaFreeHost(h_amount);
    cudaFreeHost(h_q);
    cudaFreeHost(h_k);
    cudaFree(d_q);
    cudaFree(d_k);
  }
  cudaFree(d_pos2);
  cudaFree(d_ids);
  cudaFree(d_cu);
  cudaFree(d_pos);
  cudaFree(d_start);
  cudaFree(d_amount);
  return 0;
}

int main(int argc, char** argv) {
  if (argc > 1 && strcmp(argv[1], "device") == 0) return device_run();
  return host_checks();
}
