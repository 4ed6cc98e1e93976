// C ABI of the library: argument checks on the host, then one kernel launch per
// entry point on the caller's stream. No allocation, no synchronisation.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <functional>
#include <queue>
#include <string>
#include <vector>

#include "../../include/sparse_attn.h"
#include "launch.h"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return SA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define SA_REQUIRE(cond, ...) \
  do {                        \
    if (!(cond)) return fail(SA_ERR_INVALID, __VA_ARGS__); \
  } while (0)

#define SA_REQUIRE_PTR(ptr) \
  SA_REQUIRE((ptr) != nullptr && aligned16(ptr), "%s must be a non-null 16-byte aligned pointer", #ptr)

int check_device() {
  static int cache[64];  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SA_ERR_LAUNCH, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev >= 0 && dev < 64 && cache[dev] == 1) return SA_OK;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  const bool good = major == 10 && minor == 0;
  if (dev >= 0 && dev < 64) cache[dev] = good ? 1 : 2;
  if (!good)
    return fail(SA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                major, minor);
  return SA_OK;
}

int launched(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(SA_ERR_LAUNCH, "%s: %s", what, cudaGetErrorString(e));
  return ok();
}

int check_shape(int B, int H, int Nq, int Nk, int d, int block) {
  SA_REQUIRE(B >= 0 && H >= 0 && Nq >= 0 && Nk >= 0, "B, H, Nq, Nk must be >= 0");
  SA_REQUIRE(d == 64 || d == 128, "d must be 64 or 128 (got %d)", d);
  SA_REQUIRE(block == 64 || block == 128, "block must be 64 or 128 (got %d)", block);
  SA_REQUIRE((long long)B * H <= 65535, "B*H must be <= 65535 (got %lld)", (long long)B * H);
  return SA_OK;
}

inline int cdiv(int a, int b) { return (a + b - 1) / b; }

}  // namespace

extern "C" {

const char* sparse_attn_last_error(void) { return g_last_error.c_str(); }

int sparse_attn_table_sizes(int B, int H, int Nq, int Nk, int d, int block, int order,
                            size_t sizes[7]) {
  if (int rc = check_shape(B, H, Nq, Nk, d, block)) return rc;
  SA_REQUIRE(order >= 0 && order <= 2, "order must be 0, 1 or 2");
  SA_REQUIRE(sizes != nullptr, "sizes must not be NULL");
  const size_t bh = (size_t)B * H, nqb = cdiv(Nq, block), nkb = cdiv(Nk, block);
  sizes[0] = bh * nqb * d * sizeof(float);
  sizes[1] = bh * nkb * d * sizeof(float);
  sizes[2] = bh * nkb * d * sizeof(float);
  sizes[3] = bh * 2 * nkb * d * 2;
  sizes[4] = bh * nkb * d * 2;
  sizes[5] = order >= 1 ? bh * nkb * d * d * 2 : 0;
  sizes[6] = bh * (size_t)Nk * d * 2;
  return ok();
}

int sparse_attn_pool(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int H, int Nq,
                     int Nk, int d, int block, int order, float* qbar, float* kbar_t, float* vsum,
                     uint16_t* kbar16, uint16_t* vsum16, uint16_t* M, uint16_t* v16,
                     int32_t* err_flag, void* stream) {
  if (int rc = check_shape(B, H, Nq, Nk, d, block)) return rc;
  SA_REQUIRE(order >= 0 && order <= 2, "order must be 0, 1 or 2");
  const bool do_q = q != nullptr && Nq > 0;
  if ((long long)B * H == 0 || (Nk == 0 && !do_q)) return ok();
  if (Nk > 0) {
    SA_REQUIRE_PTR(k);
    SA_REQUIRE_PTR(v);
    SA_REQUIRE_PTR(kbar_t);
    SA_REQUIRE_PTR(vsum);
    SA_REQUIRE_PTR(kbar16);
    SA_REQUIRE_PTR(vsum16);
    SA_REQUIRE_PTR(v16);
    if (order >= 1) SA_REQUIRE_PTR(M);
  }
  if (do_q) {
    SA_REQUIRE_PTR(q);
    SA_REQUIRE_PTR(qbar);
  }
  if (err_flag) SA_REQUIRE(((uintptr_t)err_flag & 3u) == 0, "err_flag must be 4-byte aligned");
  if (int rc = check_device()) return rc;
  sa::PoolArgs p{do_q ? q : nullptr, k, v, B, H, Nq, Nk, d, block, order,
                 cdiv(Nq, block), cdiv(Nk, block), qbar, kbar_t, vsum, kbar16, vsum16, M, v16,
                 0, err_flag};
  return launched(sa::launch_pool(p, static_cast<cudaStream_t>(stream)), "pool launch");
}

int sparse_attn_pool_incremental(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B,
                                 int H, int Nq, int Nk, int d, int block, int order,
                                 int kv_block_start, float* qbar, float* kbar_t, float* vsum,
                                 uint16_t* kbar16, uint16_t* vsum16, uint16_t* M, uint16_t* v16,
                                 int32_t* err_flag, void* stream) {
  if (int rc = check_shape(B, H, Nq, Nk, d, block)) return rc;
  SA_REQUIRE(order >= 0 && order <= 2, "order must be 0, 1 or 2");
  const int nkb = cdiv(Nk, block);
  SA_REQUIRE(kv_block_start >= 0 && kv_block_start <= nkb,
             "kv_block_start must be in [0, nkb] (got %d, nkb %d)", kv_block_start, nkb);
  const bool do_q = q != nullptr && Nq > 0;
  if ((long long)B * H == 0 || (kv_block_start == nkb && !do_q)) return ok();
  if (kv_block_start < nkb) {
    SA_REQUIRE_PTR(k);
    SA_REQUIRE_PTR(v);
    SA_REQUIRE_PTR(kbar_t);
    SA_REQUIRE_PTR(vsum);
    SA_REQUIRE_PTR(kbar16);
    SA_REQUIRE_PTR(vsum16);
    SA_REQUIRE_PTR(v16);
    if (order >= 1) SA_REQUIRE_PTR(M);
  }
  if (do_q) {
    SA_REQUIRE_PTR(q);
    SA_REQUIRE_PTR(qbar);
  }
  if (err_flag) SA_REQUIRE(((uintptr_t)err_flag & 3u) == 0, "err_flag must be 4-byte aligned");
  if (int rc = check_device()) return rc;
  sa::PoolArgs p{do_q ? q : nullptr, k, v, B, H, Nq, kv_block_start < nkb ? Nk : 0, d, block,
                 order, cdiv(Nq, block), nkb, qbar, kbar_t, vsum, kbar16, vsum16, M, v16,
                 kv_block_start, err_flag};
  return launched(sa::launch_pool(p, static_cast<cudaStream_t>(stream)), "pool launch");
}

int sparse_attn_route(const float* qbar, const float* kbar_t, int B, int H, int nqb, int nkb, int d,
                      int mode, int rho_num, int rho_den, float tau, float scale, int32_t* kv_idx,
                      int32_t* kv_cnt, int cap, void* stream) {
  SA_REQUIRE(B >= 0 && H >= 0 && nqb >= 0 && nkb >= 0, "B, H, nqb, nkb must be >= 0");
  SA_REQUIRE((long long)B * H <= 65535, "B*H must be <= 65535");
  SA_REQUIRE(d == 64 || d == 128, "d must be 64 or 128 (got %d)", d);
  SA_REQUIRE(mode == SA_ROUTE_TOPK || mode == SA_ROUTE_MASS, "mode must be TOPK or MASS");
  SA_REQUIRE(std::isfinite(scale), "scale must be finite");
  if ((long long)B * H * nqb == 0) return ok();
  SA_REQUIRE(nkb >= 1 && nkb <= SA_MAX_KV_BLOCKS, "nkb must be in [1, %d] (got %d)",
             SA_MAX_KV_BLOCKS, nkb);
  int keep = nkb;
  if (mode == SA_ROUTE_TOPK) {
    SA_REQUIRE(rho_num > 0 && rho_den > 0 && rho_num <= rho_den,
               "top-k needs 0 < rho_num <= rho_den (got %d/%d)", rho_num, rho_den);
    keep = (int)(((long long)rho_num * nkb + rho_den - 1) / rho_den);
    SA_REQUIRE(cap >= keep, "cap %d is below the keep count %d", cap, keep);
  } else {
    SA_REQUIRE(tau > 0.f && tau <= 1.f, "tau must be in (0, 1] (got %g)", (double)tau);
    SA_REQUIRE(cap >= nkb, "mass routing needs cap >= nkb (cap %d, nkb %d)", cap, nkb);
  }
  SA_REQUIRE_PTR(qbar);
  SA_REQUIRE_PTR(kbar_t);
  SA_REQUIRE_PTR(kv_idx);
  SA_REQUIRE_PTR(kv_cnt);
  if (int rc = check_device()) return rc;
  sa::RouteArgs p{qbar, kbar_t, B, H, nqb, nkb, d, mode, keep, tau, scale, kv_idx, kv_cnt, cap};
  return launched(sa::launch_route(p, static_cast<cudaStream_t>(stream)), "route launch");
}

int sparse_attn_route_cov(const float* qbar, const float* kbar_t, const float* cov, int B, int H,
                          int nqb, int nkb, int d, int rho_num, int rho_den, float scale,
                          int32_t* kv_idx, int32_t* kv_cnt, int cap, void* stream) {
  SA_REQUIRE(B >= 0 && H >= 0 && nqb >= 0 && nkb >= 0, "B, H, nqb, nkb must be >= 0");
  SA_REQUIRE((long long)B * H <= 65535, "B*H must be <= 65535");
  SA_REQUIRE(d == 64 || d == 128, "d must be 64 or 128 (got %d)", d);
  SA_REQUIRE(std::isfinite(scale), "scale must be finite");
  if ((long long)B * H * nqb == 0) return ok();
  SA_REQUIRE(nkb >= 1 && nkb <= SA_MAX_KV_BLOCKS, "nkb must be in [1, %d] (got %d)",
             SA_MAX_KV_BLOCKS, nkb);
  SA_REQUIRE(rho_num > 0 && rho_den > 0 && rho_num <= rho_den,
             "top-k needs 0 < rho_num <= rho_den (got %d/%d)", rho_num, rho_den);
  const int keep = (int)(((long long)rho_num * nkb + rho_den - 1) / rho_den);
  SA_REQUIRE(cap >= keep, "cap %d is below the keep count %d", cap, keep);
  SA_REQUIRE_PTR(qbar);
  SA_REQUIRE_PTR(kbar_t);
  SA_REQUIRE_PTR(cov);
  SA_REQUIRE_PTR(kv_idx);
  SA_REQUIRE_PTR(kv_cnt);
  if (int rc = check_device()) return rc;
  sa::RouteArgs p{qbar, kbar_t, B, H, nqb, nkb, d, SA_ROUTE_TOPK, keep, 1.f, scale, kv_idx, kv_cnt,
                  cap, cov};
  return launched(sa::launch_route(p, static_cast<cudaStream_t>(stream)), "route launch");
}

int sparse_attn_ear_scores(const float* qbar, const uint16_t* k, const uint16_t* v, int B, int H,
                           int nqb, int Nk, int d, int block, float scale, float* scores,
                           int32_t* err_flag, void* stream) {
  SA_REQUIRE(B >= 0 && H >= 0 && nqb >= 0 && Nk >= 0, "B, H, nqb, Nk must be >= 0");
  SA_REQUIRE((long long)B * H <= 65535, "B*H must be <= 65535");
  SA_REQUIRE(d == 64 || d == 128, "d must be 64 or 128 (got %d)", d);
  SA_REQUIRE(block == 64 || block == 128, "block must be 64 or 128 (got %d)", block);
  SA_REQUIRE(std::isfinite(scale), "scale must be finite");
  if ((long long)B * H * nqb == 0 || Nk == 0) return ok();
  const int nkb = cdiv(Nk, block);
  SA_REQUIRE(nkb <= SA_MAX_KV_BLOCKS, "nkb must be <= %d (got %d)", SA_MAX_KV_BLOCKS, nkb);
  SA_REQUIRE_PTR(qbar);
  SA_REQUIRE_PTR(k);
  SA_REQUIRE_PTR(v);
  SA_REQUIRE(scores != nullptr && ((uintptr_t)scores & 3u) == 0,
             "scores must be a non-null 4-byte aligned pointer");
  if (err_flag) SA_REQUIRE(((uintptr_t)err_flag & 3u) == 0, "err_flag must be 4-byte aligned");
  if (int rc = check_device()) return rc;
  sa::EarArgs p{qbar, k, v, B, H, Nk, d, block, nqb, nkb, scale, scores, err_flag};
  return launched(sa::launch_ear(p, static_cast<cudaStream_t>(stream)), "ear launch");
}

int sparse_attn_route_scores(const float* scores, int B, int H, int nqb, int nkb, int rho_num,
                             int rho_den, int32_t* kv_idx, int32_t* kv_cnt, int cap,
                             void* stream) {
  SA_REQUIRE(B >= 0 && H >= 0 && nqb >= 0 && nkb >= 0, "B, H, nqb, nkb must be >= 0");
  SA_REQUIRE((long long)B * H <= 65535, "B*H must be <= 65535");
  if ((long long)B * H * nqb == 0) return ok();
  SA_REQUIRE(nkb >= 1 && nkb <= SA_MAX_KV_BLOCKS, "nkb must be in [1, %d] (got %d)",
             SA_MAX_KV_BLOCKS, nkb);
  SA_REQUIRE(rho_num > 0 && rho_den > 0 && rho_num <= rho_den,
             "top-k needs 0 < rho_num <= rho_den (got %d/%d)", rho_num, rho_den);
  const int keep = (int)(((long long)rho_num * nkb + rho_den - 1) / rho_den);
  SA_REQUIRE(cap >= keep, "cap %d is below the keep count %d", cap, keep);
  SA_REQUIRE(scores != nullptr && ((uintptr_t)scores & 3u) == 0,
             "scores must be a non-null 4-byte aligned pointer");
  SA_REQUIRE_PTR(kv_idx);
  SA_REQUIRE_PTR(kv_cnt);
  if (int rc = check_device()) return rc;
  // d only picks the kernel instance; the centroid tables are not read
  sa::RouteArgs p{nullptr, nullptr, B, H, nqb, nkb, 64, SA_ROUTE_TOPK, keep, 1.f, 1.f, kv_idx,
                  kv_cnt, cap, nullptr, scores};
  return launched(sa::launch_route(p, static_cast<cudaStream_t>(stream)), "route launch");
}

int sparse_attn_hbar(const uint16_t* M, int B, int H, int nkb, int d, float* hbar,
                     uint16_t* hbar16, float* cov, void* stream) {
  SA_REQUIRE(B >= 0 && H >= 0 && nkb >= 0, "B, H, nkb must be >= 0");
  SA_REQUIRE((long long)B * H <= 65535, "B*H must be <= 65535");
  SA_REQUIRE(d == 64 || d == 128, "d must be 64 or 128 (got %d)", d);
  if ((long long)B * H == 0) return ok();
  SA_REQUIRE(nkb >= 1 && nkb <= 65535, "nkb must be in [1, 65535] (got %d)", nkb);
  SA_REQUIRE_PTR(M);
  SA_REQUIRE_PTR(hbar);
  SA_REQUIRE_PTR(hbar16);
  if (cov) SA_REQUIRE_PTR(cov);
  if (int rc = check_device()) return rc;
  sa::HbarArgs p{M, B, H, nkb, d, hbar, hbar16, cov};
  return launched(sa::launch_hbar(p, static_cast<cudaStream_t>(stream)), "hbar launch");
}

int sparse_attn_structured_mask(int B, int H, int Nq, int Nk, int block, int frame_tokens,
                                int n_frames, int window, int n_anchors, int period, int step,
                                int q_frame0, int32_t* kv_idx, int32_t* kv_cnt, int cap,
                                void* stream) {
  return sparse_attn_structured_mask_adaptive(B, H, Nq, Nk, block, frame_tokens, n_frames, window,
                                              n_anchors, period, step, q_frame0, 0, kv_idx, kv_cnt,
                                              cap, stream);
}

int sparse_attn_structured_mask_adaptive(int B, int H, int Nq, int Nk, int block, int frame_tokens,
                                         int n_frames, int window, int n_anchors, int period,
                                         int step, int q_frame0, int budget, int32_t* kv_idx,
                                         int32_t* kv_cnt, int cap, void* stream) {
  SA_REQUIRE(budget >= 0, "budget must be >= 0 (got %d)", budget);
  SA_REQUIRE(B >= 0 && H >= 0 && Nq >= 0 && Nk >= 0, "B, H, Nq, Nk must be >= 0");
  SA_REQUIRE((long long)B * H <= 65535, "B*H must be <= 65535");
  SA_REQUIRE(block == 64 || block == 128, "block must be 64 or 128 (got %d)", block);
  SA_REQUIRE(frame_tokens >= 1 && n_frames >= 1, "frame_tokens and n_frames must be >= 1");
  SA_REQUIRE(window >= 0 && n_anchors >= 0 && period >= 1 && step >= 0 && q_frame0 >= 0,
             "window, n_anchors, step, q_frame0 must be >= 0 and period >= 1");
  SA_REQUIRE((long long)Nk <= (long long)n_frames * frame_tokens,
             "Nk exceeds n_frames * frame_tokens");
  SA_REQUIRE((long long)q_frame0 * frame_tokens + Nq <= (long long)n_frames * frame_tokens,
             "the query tokens run past the last frame");
  if ((long long)B * H * Nq == 0) return ok();
  const int nkb = cdiv(Nk, block);
  SA_REQUIRE(nkb >= 1, "Nk must be >= 1");
  SA_REQUIRE(cap >= nkb, "structured mask needs cap >= nkb (cap %d, nkb %d)", cap, nkb);
  SA_REQUIRE_PTR(kv_idx);
  SA_REQUIRE_PTR(kv_cnt);
  if (int rc = check_device()) return rc;
  sa::MaskArgs p{B, H, Nq, Nk, block, frame_tokens, n_frames, window, n_anchors, period, step,
                 q_frame0, cdiv(Nq, block), nkb, kv_idx, kv_cnt, cap, budget};
  return launched(sa::launch_structured_mask(p, static_cast<cudaStream_t>(stream)), "mask launch");
}

int sparse_attn_kmeans_sizes(int B, int H, int N, int d, int C, size_t sizes[3]) {
  SA_REQUIRE(B >= 0 && H >= 0 && N >= 0, "B, H, N must be >= 0");
  SA_REQUIRE(d == 64 || d == 128, "d must be 64 or 128 (got %d)", d);
  SA_REQUIRE(C >= 1 && C <= SA_MAX_CLUSTERS, "C must be in [1, %d] (got %d)", SA_MAX_CLUSTERS, C);
  SA_REQUIRE(sizes != nullptr, "sizes must not be NULL");
  sa::kmeans_sizes(B, H, N, d, C, sizes);
  return ok();
}

int sparse_attn_kmeans(const uint16_t* x, int B, int H, int N, int d, int C, int iters,
                       double* centroids, void* cwork, int32_t* iwork, int32_t* labels,
                       int32_t* perm, int32_t* offsets, int32_t* err_flag, void* stream) {
  SA_REQUIRE(B >= 0 && H >= 0 && N >= 0, "B, H, N must be >= 0");
  SA_REQUIRE((long long)B * H <= 65535, "B*H must be <= 65535");
  SA_REQUIRE(d == 64 || d == 128, "d must be 64 or 128 (got %d)", d);
  SA_REQUIRE(C >= 1 && C <= SA_MAX_CLUSTERS, "C must be in [1, %d] (got %d)", SA_MAX_CLUSTERS, C);
  SA_REQUIRE(iters >= 0 && iters <= 1000, "iters must be in [0, 1000] (got %d)", iters);
  if ((long long)B * H == 0 || N == 0) return ok();
  SA_REQUIRE(C <= N, "C must be <= N (C %d, N %d)", C, N);
  SA_REQUIRE_PTR(x);
  SA_REQUIRE_PTR(centroids);
  SA_REQUIRE_PTR(cwork);
  SA_REQUIRE_PTR(iwork);
  SA_REQUIRE_PTR(labels);
  SA_REQUIRE_PTR(perm);
  SA_REQUIRE_PTR(offsets);
  if (err_flag) SA_REQUIRE(((uintptr_t)err_flag & 3u) == 0, "err_flag must be 4-byte aligned");
  if (int rc = check_device()) return rc;
  sa::KmeansArgs p{x, B, H, N, d, C, iters, centroids, cwork, iwork, labels, perm, offsets,
                   err_flag};
  return launched(sa::launch_kmeans(p, static_cast<cudaStream_t>(stream)), "kmeans launch");
}

int sparse_attn_kmeans_noalloc(const uint16_t* x, int B, int H, int N, int d, int C, int iters,
                               double* centroids, int32_t* labels, int32_t* perm,
                               int32_t* offsets, int32_t* err_flag, void* stream) {
  SA_REQUIRE(B >= 0 && H >= 0 && N >= 0, "B, H, N must be >= 0");
  SA_REQUIRE(d == 64 || d == 128, "d must be 64 or 128 (got %d)", d);
  SA_REQUIRE(C >= 1 && C <= SA_MAX_CLUSTERS, "C must be in [1, %d] (got %d)", SA_MAX_CLUSTERS, C);
  size_t sizes[3];
  sa::kmeans_sizes(B, H, N, d, C, sizes);
  const size_t cw = (sizes[1] + 255) & ~(size_t)255;
  SA_REQUIRE(cw + sizes[2] <= sa::kKmeansScratchBytes,
             "problem needs %zu scratch bytes; the built-in buffer holds %zu (use sparse_attn_kmeans)",
             cw + sizes[2], sa::kKmeansScratchBytes);
  if ((long long)B * H == 0 || N == 0) return sparse_attn_kmeans(x, B, H, N, d, C, iters, centroids,
                                                                 nullptr, nullptr, labels, perm,
                                                                 offsets, err_flag, stream);
  if (int rc = check_device()) return rc;
  void* addr = nullptr;
  const cudaError_t e = sa::kmeans_scratch(&addr);
  if (e != cudaSuccess)
    return fail(SA_ERR_LAUNCH, "cudaGetSymbolAddress of the built-in scratch buffer: %s",
                cudaGetErrorString(e));
  uint8_t* scratch = static_cast<uint8_t*>(addr);
  return sparse_attn_kmeans(x, B, H, N, d, C, iters, centroids, scratch,
                            reinterpret_cast<int32_t*>(scratch + cw), labels, perm, offsets,
                            err_flag, stream);
}

int sparse_attn_permute_rows(const void* src, const int32_t* perm, int B, int H, int N,
                             int row_bytes, int gather, void* dst, void* stream) {
  SA_REQUIRE(B >= 0 && H >= 0 && N >= 0, "B, H, N must be >= 0");
  SA_REQUIRE(row_bytes > 0 && row_bytes % 16 == 0, "row_bytes must be a positive multiple of 16");
  SA_REQUIRE(gather == 0 || gather == 1, "gather must be 0 or 1");
  if ((long long)B * H * N == 0) return ok();
  SA_REQUIRE_PTR(src);
  SA_REQUIRE_PTR(perm);
  SA_REQUIRE_PTR(dst);
  SA_REQUIRE(src != dst, "src and dst must not be the same buffer");
  if (int rc = check_device()) return rc;
  sa::PermuteArgs p{src, perm, B, H, N, row_bytes, gather != 0, dst};
  return launched(sa::launch_permute_rows(p, static_cast<cudaStream_t>(stream)), "permute launch");
}

int sparse_attn_wait_selftest(int32_t* err_flag, int rounds, int32_t* waited, void* stream) {
  SA_REQUIRE(rounds >= 1 && rounds <= (1 << 20), "rounds must be in [1, 2^20] (got %d)", rounds);
  SA_REQUIRE(err_flag != nullptr && ((uintptr_t)err_flag & 3u) == 0,
             "err_flag must be a non-null 4-byte aligned pointer");
  SA_REQUIRE(waited != nullptr && ((uintptr_t)waited & 3u) == 0,
             "waited must be a non-null 4-byte aligned pointer");
  if (int rc = check_device()) return rc;
  return launched(sa::launch_wait_selftest(err_flag, (uint32_t)rounds, waited,
                                           static_cast<cudaStream_t>(stream)),
                  "selftest launch");
}

int sparse_attn_forward(const uint16_t* q, const uint16_t* k, const uint16_t* v16,
                        const uint16_t* kbar16, const uint16_t* vsum16, const uint16_t* M,
                        const int32_t* kv_idx, const int32_t* kv_cnt, int cap, int B, int H, int Nq,
                        int Nk, int d, int block, int order, float scale, void* out, int out_dtype,
                        int32_t* err_flag, void* stream) {
  if (int rc = check_shape(B, H, Nq, Nk, d, block)) return rc;
  SA_REQUIRE(order >= 0 && order <= 2, "order must be 0, 1 or 2");
  SA_REQUIRE(out_dtype == SA_OUT_F32 || out_dtype == SA_OUT_BF16, "out_dtype must be F32 or BF16");
  SA_REQUIRE(std::isfinite(scale), "scale must be finite");
  if ((long long)B * H * Nq == 0) return ok();
  SA_REQUIRE(Nk >= 1, "Nk must be >= 1 when there are queries");
  const int nkb = cdiv(Nk, block);
  SA_REQUIRE(nkb <= SA_MAX_KV_BLOCKS, "nkb must be <= %d (got %d)", SA_MAX_KV_BLOCKS, nkb);
  SA_REQUIRE(cap >= 0, "cap must be >= 0");
  SA_REQUIRE_PTR(q);
  SA_REQUIRE_PTR(k);
  SA_REQUIRE_PTR(v16);
  SA_REQUIRE_PTR(kbar16);
  SA_REQUIRE_PTR(vsum16);
  if (order >= 1) SA_REQUIRE_PTR(M);
  SA_REQUIRE_PTR(kv_idx);
  SA_REQUIRE_PTR(kv_cnt);
  SA_REQUIRE_PTR(out);
  if (err_flag) SA_REQUIRE(((uintptr_t)err_flag & 3u) == 0, "err_flag must be 4-byte aligned");
  if (int rc = check_device()) return rc;
  sa::ForwardArgs p{q, k, v16, kbar16, vsum16, order >= 1 ? M : nullptr, kv_idx, kv_cnt, cap,
                    B, H, Nq, Nk, d, block, order, cdiv(Nq, block), nkb, scale, out, out_dtype,
                    err_flag, 1, nullptr};
  return launched(sa::launch_forward(p, static_cast<cudaStream_t>(stream)), "forward launch");
}

int sparse_attn_forward_work_bytes(int B, int H, int Nq, int d, int splits, size_t* bytes) {
  if (int rc = check_shape(B, H, Nq, 1, d, 64)) return rc;
  SA_REQUIRE(splits >= 1 && splits <= SA_MAX_SPLITS, "splits must be in [1, %d] (got %d)",
             SA_MAX_SPLITS, splits);
  SA_REQUIRE(bytes != nullptr, "bytes must be non-null");
  *bytes = sa::forward_work_floats(B, H, Nq, d, splits) * sizeof(float);
  return ok();
}

int sparse_attn_forward_split_plan(int B, int H, int Nq, int Nk, int d, int block, int sms,
                                   int* splits, size_t* work_bytes) {
  if (int rc = check_shape(B, H, Nq, Nk, d, block)) return rc;
  SA_REQUIRE(splits != nullptr && work_bytes != nullptr, "splits and work_bytes must be non-null");
  SA_REQUIRE(sms >= 0, "sms must be >= 0");
  if (sms == 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(SA_ERR_LAUNCH, "SM count: %s", cudaGetErrorString(e));
  }
  *splits = 1;
  *work_bytes = 0;
  const long long bh = (long long)B * H;
  if (bh == 0 || Nq == 0 || Nk == 0) return ok();
  // CTAs of the unsplit grid: per (batch, head), the full pairs of 128-row tiles and a
  // last pair with one or two tiles (cost 1/2 or 1 of a full one).
  const int nx = cdiv(Nq, 256), ntl = cdiv(cdiv(Nk, block), 64);
  const int last_tiles = cdiv(Nq - (nx - 1) * 256, 128);
  if (bh * nx >= 8LL * sms) return ok();  // many waves: the last one costs little
  // Model: every split CTA costs 1/S of its unsplit cost plus a fixed setup and drain
  // (about eight work items against ~nkb items per unsplit CTA); CTAs start in grid order
  // on the first SM that is free. The time of a split count is the makespan, plus a
  // small charge per split for the merge.
  const double setup = 8.0 / std::max(1, cdiv(Nk, block));
  auto makespan = [&](int S) {
    std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
    for (int i = 0; i < sms; ++i) free_at.push(0.0);
    double end = 0.0;
    auto run = [&](double cost, long long n) {
      for (long long i = 0; i < n; ++i) {
        const double t = free_at.top() + cost;
        free_at.pop();
        free_at.push(t);
        end = std::max(end, t);
      }
    };
    run(1.0 / S + setup, bh * (nx - 1) * S);
    run(0.5 * last_tiles / S + setup, bh * S);
    return end + 0.003 * (S - 1);
  };
  double best = makespan(1);
  for (int S = 2; S <= std::min(ntl, SA_MAX_SPLITS); ++S) {
    if (bh * nx * S > 400000) break;
    const double t = makespan(S);
    if (t < 0.97 * best) {
      best = t;
      *splits = S;
    }
  }
  *work_bytes = sa::forward_work_floats(B, H, Nq, d, *splits) * sizeof(float);
  return ok();
}

int sparse_attn_forward_split(const uint16_t* q, const uint16_t* k, const uint16_t* v16,
                              const uint16_t* kbar16, const uint16_t* vsum16, const uint16_t* M,
                              const int32_t* kv_idx, const int32_t* kv_cnt, int cap, int B, int H,
                              int Nq, int Nk, int d, int block, int order, float scale, int splits,
                              float* work, void* out, int out_dtype, int32_t* err_flag,
                              void* stream) {
  SA_REQUIRE(splits >= 1 && splits <= SA_MAX_SPLITS, "splits must be in [1, %d] (got %d)",
             SA_MAX_SPLITS, splits);
  if (splits == 1)
    return sparse_attn_forward(q, k, v16, kbar16, vsum16, M, kv_idx, kv_cnt, cap, B, H, Nq, Nk, d,
                               block, order, scale, out, out_dtype, err_flag, stream);
  if (int rc = check_shape(B, H, Nq, Nk, d, block)) return rc;
  SA_REQUIRE(order >= 0 && order <= 2, "order must be 0, 1 or 2");
  SA_REQUIRE(out_dtype == SA_OUT_F32 || out_dtype == SA_OUT_BF16, "out_dtype must be F32 or BF16");
  SA_REQUIRE(std::isfinite(scale), "scale must be finite");
  if ((long long)B * H * Nq == 0) return ok();
  SA_REQUIRE(Nk >= 1, "Nk must be >= 1 when there are queries");
  const int nkb = cdiv(Nk, block);
  SA_REQUIRE(nkb <= SA_MAX_KV_BLOCKS, "nkb must be <= %d (got %d)", SA_MAX_KV_BLOCKS, nkb);
  SA_REQUIRE(cap >= 0, "cap must be >= 0");
  SA_REQUIRE_PTR(q);
  SA_REQUIRE_PTR(k);
  SA_REQUIRE_PTR(v16);
  SA_REQUIRE_PTR(kbar16);
  SA_REQUIRE_PTR(vsum16);
  if (order >= 1) SA_REQUIRE_PTR(M);
  SA_REQUIRE_PTR(kv_idx);
  SA_REQUIRE_PTR(kv_cnt);
  SA_REQUIRE_PTR(work);
  SA_REQUIRE_PTR(out);
  if (err_flag) SA_REQUIRE(((uintptr_t)err_flag & 3u) == 0, "err_flag must be 4-byte aligned");
  if (int rc = check_device()) return rc;
  sa::ForwardArgs p{q, k, v16, kbar16, vsum16, order >= 1 ? M : nullptr, kv_idx, kv_cnt, cap,
                    B, H, Nq, Nk, d, block, order, cdiv(Nq, block), nkb, scale, out, out_dtype,
                    err_flag, splits, work};
  return launched(sa::launch_forward(p, static_cast<cudaStream_t>(stream)), "forward launch");
}

}  // extern "C"
