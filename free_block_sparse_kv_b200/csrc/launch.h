// Host-side launch interfaces between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

struct PoolArgs {
  const uint16_t *q, *k, *v;
  int B, H, Nq, Nk, d, block, order, nqb, nkb;
  float *qbar, *kbar_t, *vsum;
  uint16_t *kbar16, *vsum16, *M, *v16;
  int j0 = 0;  // first KV block pooled (the tables of blocks < j0 are left as they are)
  int32_t* err_flag = nullptr;  // SA_FLAG_RANGE when an fp16 value does not fit
};

struct RouteArgs {
  const float *qbar, *kbar_t;
  int B, H, nqb, nkb, d, mode, keep;
  float tau, scale;
  int32_t *kv_idx, *kv_cnt;
  int cap;
  const float* cov = nullptr;     // per-block covariance norms: score += ln cov_j (top-k)
  const float* scores = nullptr;  // [B*H][nqb][nkb] precomputed scores (top-k over them)
};

struct EarArgs {
  const float* qbar;
  const uint16_t *k, *v;
  int B, H, Nk, d, block, nqb, nkb;
  float scale;
  float* scores;
  int32_t* err_flag;
  int run = 0;  // key blocks per CTA (0: default)
};

struct HbarArgs {
  const uint16_t* M;
  int B, H, nkb, d;
  float* hbar;
  uint16_t* hbar16;
  float* cov;
};

struct MaskArgs {
  int B, H, Nq, Nk, block, frame_tokens, n_frames, window, n_anchors, period, step, q_frame0;
  int nqb, nkb;
  int32_t *kv_idx, *kv_cnt;
  int cap;
  int budget = 0;  // > 0: adaptive windows reaching |A(t)| = budget frames
};

struct ForwardArgs {
  const uint16_t *q, *k, *v, *kbar16, *vsum16, *M;
  const int32_t *kv_idx, *kv_cnt;
  int cap, B, H, Nq, Nk, d, block, order, nqb, nkb;
  float scale;
  void* out;
  int out_dtype;
  int32_t* err_flag;
  int splits;   // key-range splits (1: none)
  float* work;  // splits > 1: partial results, forward_work_floats(...) floats
};

// Floats of partial results a forward with `splits` key-range splits needs: per split and
// query row, the row's D accumulators and its (max, sum) pair.
inline size_t forward_work_floats(int B, int H, int Nq, int d, int splits) {
  return splits > 1 ? (size_t)splits * B * H * Nq * (size_t)(d + 2) : 0;
}

struct KmeansArgs {
  const uint16_t* x;
  int B, H, N, d, C, iters;
  double* cent;
  void* cwork;
  int32_t* iwork;
  int32_t *labels, *perm, *offsets;
  int32_t* err_flag;
  // carved from cwork / iwork by the launcher
  uint16_t* pieces = nullptr;
  float* cnorm = nullptr;
  int32_t *counts = nullptr, *amb_list = nullptr, *amb_cnt = nullptr;
};

struct PermuteArgs {
  const void* src;
  const int32_t* perm;
  int B, H, N, row_bytes;
  bool gather;
  void* dst;
};

// Byte offsets of launch_kmeans's work buffers in cwork and iwork, and the two ends.
struct KmeansLayout {
  size_t pieces, cnorm, part, cwork_end;
  size_t counts, amb_list, amb_cnt, seg_off, iwork_end;
};
KmeansLayout kmeans_layout(int B, int H, int N, int d, int C);
void kmeans_sizes(int B, int H, int N, int d, int C, size_t sizes[3]);
constexpr size_t kKmeansScratchBytes = (size_t)32 << 20;  // per device, for the no-alloc call
cudaError_t kmeans_scratch(void** addr);  // device address of that buffer, current device
cudaError_t launch_kmeans(const KmeansArgs& p, cudaStream_t st);
cudaError_t launch_permute_rows(const PermuteArgs& p, cudaStream_t st);
cudaError_t launch_wait_selftest(int32_t* err_flag, uint32_t rounds, int32_t* waited,
                                 cudaStream_t st);
cudaError_t launch_pool(const PoolArgs& p, cudaStream_t st);
cudaError_t launch_route(const RouteArgs& p, cudaStream_t st);
cudaError_t launch_structured_mask(const MaskArgs& p, cudaStream_t st);
cudaError_t launch_forward(const ForwardArgs& p, cudaStream_t st);
cudaError_t launch_hbar(const HbarArgs& p, cudaStream_t st);
cudaError_t launch_ear(const EarArgs& p, cudaStream_t st);

}  // namespace sa
