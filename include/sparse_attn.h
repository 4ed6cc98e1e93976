/*
 * sparse_attn.h - C ABI of the block-sparse attention library with compensation
 * for skipped blocks, for NVIDIA B200 (sm_100a).
 *
 * The operation. Per (batch b, head h), with Q [Nq, d] and K, V [Nk, d] split into
 * blocks of `block` tokens (the last block may be partial, holding n_j tokens):
 *   - every KV block j is pooled into its centroid kbar_j = mean K, its value sum
 *     S_j = sum V and (first order) M_j = sum_r (k_r - kbar_j) v_r^T;
 *   - every query block i keeps a set of KV blocks, chosen from the pooled scores
 *     scale * qbar_i . kbar_j (top-rho or covering mass tau), or from a frame
 *     geometry (local window plus rotating anchor frames);
 *   - the output o_t = N_t / D_t sums exact softmax terms over the tokens of kept
 *     blocks and, for every skipped block j, alpha_tj * (S_j + [order 1] scale *
 *     q_t M_j) in the numerator and alpha_tj * n_j in the denominator, with
 *     alpha_tj = exp(scale * q_t . kbar_j): all inside one softmax.
 * Sources: "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
 * Transformers" §2 (Algorithme Central: o_t = N_t / D_t, the numerator N_t,
 * alpha_{t,j}; Cohérence de Normalisation; Implémentation Matérielle);
 * "LVSA: Training-Free Sparse Attention for Long Video Diffusion" §2 (Mécanisme
 * Central: A(t) = G u W(t), rotating anchors); "SVG-EAR: Parameter-Free Linear
 * Compensation for Sparse Video Generation via Error-aware Routing" §2 (centroid
 * substitution; query centroids as routing proxies).
 *
 * Conventions for every entry point.
 *   - bf16 and fp16 tensors are passed as pointers to their 16-bit patterns (uint16_t).
 *   - Tensors are dense and contiguous in the layout stated for each argument,
 *     d innermost. Every device pointer must be 16-byte aligned.
 *   - The caller allocates and owns every buffer. The library never allocates,
 *     frees or synchronises; all work is enqueued on `stream` (a cudaStream_t,
 *     NULL for the legacy default stream) in call order.
 *   - Supported shapes: d in {64, 128}; block in {64, 128}; B, H >= 0; Nq, Nk >= 0.
 *     A call with an empty problem (B*H*Nq == 0) returns SA_OK and does nothing.
 *     Nq = 0 with Nk > 0 and the reverse are both empty for the forward.
 *   - Return value: SA_OK, or an error code below; the calling thread's last
 *     error message is then available from sparse_attn_last_error(). Argument
 *     errors are found on the host before anything is enqueued.
 */
#ifndef SPARSE_ATTN_H_
#define SPARSE_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  SA_OK = 0,
  SA_ERR_INVALID = 1,      /* bad shape, null or misaligned pointer, capacity too small */
  SA_ERR_LAUNCH = 2,       /* a CUDA launch or runtime call failed */
  SA_ERR_TIMEOUT = 3,      /* a bounded device wait gave up (reported through err_flag) */
  SA_ERR_UNSUPPORTED = 4,  /* the current device is not sm_100 */
  SA_ERR_RANGE = 5         /* a pooled fp16 table value does not fit (reported through err_flag) */
};

/* Bit set in err_flag by the pool when a value of its fp16 outputs (V copy, value sums,
 * M_j) would round to infinity (|x| >= 65520). The other bits of err_flag mark bounded
 * device waits that gave up (SA_ERR_TIMEOUT). */
#define SA_FLAG_RANGE (1 << 20)

enum { SA_ROUTE_TOPK = 0, SA_ROUTE_MASS = 1 };
enum { SA_OUT_F32 = 0, SA_OUT_BF16 = 1 };

/* Largest number of KV blocks per head that routing and the forward accept. */
#define SA_MAX_KV_BLOCKS 2048
#define SA_MAX_CLUSTERS 4096
#define SA_MAX_SPLITS 16

/*
 * Byte sizes of the pooled tables for a problem, written to sizes[0..6] in the
 * order qbar, kbar_t, vsum, kbar16, vsum16, M (0 when order == 0), v16. Order 2 needs
 * the M table like order 1; its global tables (see sparse_attn_hbar) take
 * B*H*d*d*4 (hbar), B*H*d*d*2 (hbar16) and B*H*nkb*4 (cov) bytes.
 * nqb = ceil(Nq / block), nkb = ceil(Nk / block).
 */
int sparse_attn_table_sizes(int B, int H, int Nq, int Nk, int d, int block, int order,
                            size_t sizes[7]);

/*
 * Pooling (PISA §2 Implémentation Matérielle, pre-computation step; the per-block
 * first-order matrix of the Taylor expansion about kbar_j; SVG-EAR §2 B query
 * centroids). One pass over Q, K and V.
 *   q       [B,H,Nq,d] bf16, may be NULL (then qbar is not written and may be NULL)
 *   k, v    [B,H,Nk,d] bf16
 *   order   0, 1 or 2; with 1 or 2, M is written and must not be NULL
 *   qbar    [B,H,nqb,d]  fp32   mean of each query block's rows
 *   kbar_t  [B,H,d,nkb]  fp32   block centroids, dim-major (routing reads it)
 *   vsum    [B,H,nkb,d]  fp32   value sums S_j
 *   kbar16  [B,H,2,nkb,d] bf16  centroids as hi + lo: plane 0 = rn(kbar), plane 1 =
 *                               rn(kbar - hi); hi + lo carries ~16 significant bits
 *                               (forward reads it)
 *   vsum16  [B,H,nkb,d]  fp16   value sums, rounded to nearest (forward reads it)
 *   M       [B,H,nkb,d,d] fp16  M_j[a][c] = sum_r (k_r[a] - kbar_j[a]) v_r[c],
 *                               a = key dim (rows), c = value dim; fp32 accumulate
 *   v16     [B,H,Nk,d]   fp16   V converted to fp16 (exact for |v| in the fp16
 *                               normal range)
 *   err_flag  optional device int32 (4-byte aligned): SA_FLAG_RANGE is ORed into it
 *             when a value of vsum16, M or v16 does not fit in fp16 (|x| >= 65520; the
 *             table then holds an infinity and the forward's output is not valid), other
 *             bits when a bounded device wait gave up. NULL: nothing is reported.
 * Precision departs from a bf16 table format on purpose: vsum16, M and v16 are IEEE
 * fp16 (11-bit significand against bf16's 8), because the forward multiplies them by
 * probabilities (also fp16) on the tensor cores, and bf16 probabilities would put up to
 * ~2^-8 relative error on single dominant terms; fp16's narrower range is what
 * err_flag guards. The centroids are two bf16 planes (hi + lo, ~16 significant bits)
 * because they meet the bf16 queries in the centroid logits. Logits use the bf16 Q
 * against the bf16 K as given (kept tokens) or against both centroid planes (skipped
 * blocks). Means of a partial last block use its true token count.
 * One launch (one persistent CTA per SM).
 */
int sparse_attn_pool(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     int B, int H, int Nq, int Nk, int d, int block, int order,
                     float* qbar, float* kbar_t, float* vsum,
                     uint16_t* kbar16, uint16_t* vsum16, uint16_t* M, uint16_t* v16,
                     int32_t* err_flag, void* stream);

/*
 * Incremental pooling for a growing KV cache (an autoregressive world model attends a new
 * chunk of frames to every earlier frame): as sparse_attn_pool, but only the KV blocks
 * kv_block_start .. nkb-1 are pooled and written (kbar_t, vsum, kbar16, vsum16, M rows and
 * the v16 tokens of those blocks); the tables of the earlier blocks are left as an earlier
 * call wrote them. Query blocks are pooled as usual when q is given. Pooling blocks
 * [0, s) in one call and [s, nkb) in another gives the tables of one full call, bit for
 * bit. 0 <= kv_block_start <= nkb. For order 2, sparse_attn_hbar is run again afterwards
 * (it reads every M_j).
 */
int sparse_attn_pool_incremental(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 int B, int H, int Nq, int Nk, int d, int block, int order,
                                 int kv_block_start, float* qbar, float* kbar_t, float* vsum,
                                 uint16_t* kbar16, uint16_t* vsum16, uint16_t* M, uint16_t* v16,
                                 int32_t* err_flag, void* stream);

/*
 * Routing (PISA §2 top-k choice of the critical blocks; SVG-EAR §2 B pooled
 * proxies). Scores s_ij = scale * qbar_i . kbar_j in fp32; blocks are ordered by
 * (s descending, j ascending).
 *   qbar    [B,H,nqb,d] fp32;  kbar_t [B,H,d,nkb] fp32 (as written by the pool)
 *   mode    SA_ROUTE_TOPK: keep the first ceil(rho_num * nkb / rho_den) blocks
 *                          (integer arithmetic; 0 < rho_num <= rho_den)
 *           SA_ROUTE_MASS: keep the shortest prefix whose softmax(s_i.) mass is
 *                          >= tau (0 < tau <= 1)
 *   kv_idx  [B,H,nqb,cap] int32  kept block indices of each query block, ascending;
 *                                entries past kv_cnt are left untouched
 *   kv_cnt  [B,H,nqb]     int32  number of kept blocks
 *   cap     >= the keep count for TOPK, >= nkb for MASS
 * nkb <= SA_MAX_KV_BLOCKS.
 */
int sparse_attn_route(const float* qbar, const float* kbar_t,
                      int B, int H, int nqb, int nkb, int d,
                      int mode, int rho_num, int rho_den, float tau, float scale,
                      int32_t* kv_idx, int32_t* kv_cnt, int cap, void* stream);

/*
 * Global first-order statistic (PISA §2 Algorithme Central: Hbar, the mean of the
 * per-block first-order matrices over all blocks, used in place of each skipped
 * block's own matrix) and per-block covariance norms (PISA §2 Routage Sensible à la
 * Covariance: ||H_j - Hbar||, here the 2-norm of the matrix entries).
 *   M       [B,H,nkb,d,d] fp16, as written by the pool with order 1 or 2
 *   hbar    [B,H,d,d] fp32    Hbar = (1/nkb) sum_j M_j (fp32 accumulate)
 *   hbar16  [B,H,d,d] fp16    Hbar rounded to nearest (the forward's order-2 operand)
 *   cov     [B,H,nkb] fp32    sqrt(sum over entries of (M_j - Hbar)^2); may be NULL
 * Two launches on the stream (mean, then norms).
 */
int sparse_attn_hbar(const uint16_t* M, int B, int H, int nkb, int d, float* hbar,
                     uint16_t* hbar16, float* cov, void* stream);

/*
 * Covariance-aware top-k (PISA §2 Routage Sensible à la Covariance). As
 * sparse_attn_route with SA_ROUTE_TOPK, on the scores
 *   s'_ij = scale * qbar_i . kbar_j + ln cov_j
 * (fp32): the log of the first-order error bound alpha_ij * scale * |qbar_i| *
 * ||H_j - Hbar|| of the hybrid order, up to a term that is the same for every
 * block of the row.
 *   cov     [B,H,nkb] fp32, as written by sparse_attn_hbar (positive)
 */
int sparse_attn_route_cov(const float* qbar, const float* kbar_t, const float* cov,
                          int B, int H, int nqb, int nkb, int d, int rho_num, int rho_den,
                          float scale, int32_t* kv_idx, int32_t* kv_cnt, int cap,
                          void* stream);

/*
 * Error-aware routing scores (SVG-EAR §2 B, Routage Sensible à l'Erreur: the squared
 * error of the centroid approximation per key block, query centroids as proxies,
 * normalised by the block's size; §2 C: computed in one streaming pass, no logit is
 * written). For query centroid i and key block j with n_j tokens:
 *   s_r = scale * qbar_i . k_r (r in block j),  s_c = mean_r s_r = scale * qbar_i . kbar_j,
 *   err_ij = || sum_r (exp(s_r) - exp(s_c)) v_r ||^2,
 *   scores[i][j] = ln(err_ij / n_j)   (-inf when err_ij = 0).
 * Computed on the tensor cores with fp32 accumulation: qbar as two bf16 pieces
 * (about 16 significant bits), the weight differences as two bf16 pieces (the top
 * 16 bits of each), every weight relative to the block's largest logit.
 *   qbar      [B,H,nqb,d] fp32 (as written by the pool)
 *   k, v      [B,H,Nk,d]  bf16, as for the pool
 *   scores    [B,H,nqb,nkb] fp32, nkb = ceil(Nk / block); every entry is written
 *   err_flag  optional int32 (4-byte aligned): nonzero after a launch whose waits
 *             gave up (that launch's scores are then undefined)
 * k, v and qbar must be 16-byte aligned. One launch; nkb <= SA_MAX_KV_BLOCKS.
 */
int sparse_attn_ear_scores(const float* qbar, const uint16_t* k, const uint16_t* v,
                           int B, int H, int nqb, int Nk, int d, int block, float scale,
                           float* scores, int32_t* err_flag, void* stream);

/*
 * Top-k over precomputed block scores (the greedy error-per-cost choice of SVG-EAR
 * §2 B under a density budget read as a block count): keeps, per query block, the
 * first ceil(rho_num * nkb / rho_den) blocks in the order (score descending, j
 * ascending); -inf scores sort last. Same list format as sparse_attn_route.
 *   scores  [B,H,nqb,nkb] fp32, e.g. from sparse_attn_ear_scores (no NaN)
 */
int sparse_attn_route_scores(const float* scores, int B, int H, int nqb, int nkb,
                             int rho_num, int rho_den, int32_t* kv_idx, int32_t* kv_cnt,
                             int cap, void* stream);

/*
 * Cluster-permuted token layout (SVG-EAR §2 A: query and key tokens grouped into
 * semantic clusters by k-means; "Partition the Support, Reconstruct the Residual"
 * (SparsePR) §2 C: tokens permuted into contiguous group-major layouts before the
 * block-sparse attention).
 *
 * sparse_attn_kmeans_sizes: byte sizes of the buffers sparse_attn_kmeans needs:
 *   sizes[0] centroids (fp64), sizes[1] cwork, sizes[2] iwork.
 *
 * sparse_attn_kmeans: Lloyd's k-means on the rows of x per (b, h), then the stable
 * group-major order of the final labels.
 *   x          [B,H,N,d] bf16 (Q or K as given), 16-byte aligned
 *   C          clusters, 1 <= C <= min(N, SA_MAX_CLUSTERS); iters update steps, 0..1000
 *   centroids  [B,H,C,d] fp64, out: the final centroids
 *   cwork, iwork  scratch of sizes[1] and sizes[2] bytes (16-byte aligned), contents
 *              undefined on return
 *   labels     [B,H,N] int32, out: cluster of every token after the final assignment
 *   perm       [B,H,N] int32, out: perm[p] = original index of the token at position p
 *              (tokens by cluster, then by original index)
 *   offsets    [B,H,C+1] int32, out: positions offsets[m] .. offsets[m+1]-1 hold cluster m
 *   err_flag   optional int32: nonzero after a launch whose waits gave up
 * Iteration: every centroid starts at token floor(m N / C); each token goes to its
 * nearest centroid (squared Euclidean distance, ties to the lowest index), each centroid
 * with members moves to their mean (fp64; the others stay); after `iters` updates the
 * tokens are assigned once more. The assignment runs on the tensor cores (fp32 scores
 * from a two-piece bf16 split of the fp64 centroids); a token whose two best scores lie
 * within that arithmetic's error bound is decided again in fp64. 7 + 8 * iters
 * launches on the stream.
 *
 * sparse_attn_permute_rows: rows of row_bytes bytes (a multiple of 16) per (b, h);
 *   gather = 1: dst[p] = src[perm[p]] (into the clustered order);
 *   gather = 0: dst[perm[p]] = src[p] (back to the original order).
 * src and dst must not overlap. One launch.
 */
int sparse_attn_kmeans_sizes(int B, int H, int N, int d, int C, size_t sizes[3]);
int sparse_attn_kmeans(const uint16_t* x, int B, int H, int N, int d, int C, int iters,
                       double* centroids, void* cwork, int32_t* iwork, int32_t* labels,
                       int32_t* perm, int32_t* offsets, int32_t* err_flag, void* stream);
int sparse_attn_permute_rows(const void* src, const int32_t* perm, int B, int H, int N,
                             int row_bytes, int gather, void* dst, void* stream);

/*
 * sparse_attn_kmeans_noalloc: sparse_attn_kmeans without caller scratch. The pages have
 * no counterpart for this call; it is an interface convenience for callers that cannot
 * allocate device memory. cwork and iwork come from one built-in 32 MiB buffer per
 * device (module global memory, obtained with cudaGetSymbolAddress); problems whose
 * sizes[1] (rounded up to 256 bytes) + sizes[2] exceed it return SA_ERR_INVALID before
 * anything is enqueued. The buffer is shared by every call on the device: calls must be
 * ordered (one stream, or synchronised), never concurrent. Results equal
 * sparse_attn_kmeans's bit for bit. Every call looks up the buffer's address on the
 * current device (cudaGetSymbolAddress; a failed lookup returns SA_ERR_LAUNCH with the
 * runtime's message and leaves no pending runtime error); the first lookup on a device
 * may load the library's module there, so make the first call on each device outside
 * any stream capture.
 */
int sparse_attn_kmeans_noalloc(const uint16_t* x, int B, int H, int N, int d, int C, int iters,
                               double* centroids, int32_t* labels, int32_t* perm,
                               int32_t* offsets, int32_t* err_flag, void* stream);

/*
 * Structured mask (LVSA §2 Mécanisme Central). Tokens are frame-major with
 * frame_tokens tokens per frame; query token t lies in frame
 * q_frame0 + t / frame_tokens and key token r in frame r / frame_tokens.
 * At denoising step `step` the anchor frames are
 *   G = { (step mod period) + period * m : m = 0 .. n_anchors-1 } (those < n_frames),
 * and query frame f attends A(f) = G u { f-window .. f+window } (inside the video).
 * KV block j is kept for query block i when some query token of i and some key
 * token of j have frames (f, g) with g in A(f). Same list format as routing;
 * cap >= nkb. Every (b, h) gets the same lists.
 */
int sparse_attn_structured_mask(int B, int H, int Nq, int Nk, int block,
                                int frame_tokens, int n_frames, int window,
                                int n_anchors, int period, int step, int q_frame0,
                                int32_t* kv_idx, int32_t* kv_cnt, int cap, void* stream);

/*
 * Structured mask with extended adaptive windows (LVSA §2 Fenêtres Adaptatives
 * Étendues). As sparse_attn_structured_mask, but each query frame's window
 * { f-window .. f+window } (inside the video) grows one frame at a time, alternately
 * after and before it (a side at the edge of the video is skipped), while
 * |G u window| < budget, so that overlaps with the anchors and clipping at the edges
 * are made up: |A(f)| = max(|G u {f-window .. f+window}|, min(budget, n_frames)).
 * budget = 0 gives sparse_attn_structured_mask.
 */
int sparse_attn_structured_mask_adaptive(int B, int H, int Nq, int Nk, int block,
                                         int frame_tokens, int n_frames, int window,
                                         int n_anchors, int period, int step, int q_frame0,
                                         int budget, int32_t* kv_idx, int32_t* kv_cnt, int cap,
                                         void* stream);

/*
 * Self-test of the device-side failure path: one CTA waits on an mbarrier that nothing
 * arrives on, with the library's bounded wait (`rounds` try_wait rounds of about 1 us
 * each, 1 <= rounds <= 2^20). The wait gives up, sets bit 0 of *err_flag (device int32)
 * and writes 0 to *waited (device int32; 1 would mean the wait had completed). The
 * context stays usable. One launch.
 */
int sparse_attn_wait_selftest(int32_t* err_flag, int rounds, int32_t* waited, void* stream);

/*
 * Forward (PISA §2 Algorithme Central and Implémentation Matérielle, phases 1-3,
 * with the first-order term per block, or global with order 2). For each query
 * row t of query block i:
 *   exact logits    scale * q_t . k_r   for the tokens r of the kept blocks of i
 *   centroid logits scale * q_t . kbar_j for the other blocks j
 *   N_t = sum_r e^(l_r - m) v_r + sum_j e^(c_j - m) (S_j + [order 1] scale * q_t M_j
 *                                                      + [order 2] scale * q_t Hbar)
 *   D_t = sum_r e^(l_r - m)     + sum_j e^(c_j - m) n_j
 *   o_t = N_t / D_t
 *   q, k              [B,H,Nq,d] / [B,H,Nk,d] bf16, as for the pool
 *   v16, kbar16, vsum16  as written by the pool. The forward reads the pool's fp16 copy
 *                     of V rather than V itself: the exact value products multiply fp16
 *                     probabilities (bf16 ones would carry ~2^-8 relative error on a
 *                     dominant term), and a tensor-core product takes one 16-bit type for
 *                     both operands.
 *   M                 order 1: the pool's M table; order 2: hbar16 [B,H,d,d] from
 *                     sparse_attn_hbar; order 0: NULL
 *   kv_idx, kv_cnt    as written by routing or the structured mask: indices of
 *                     each row must be distinct and < nkb; entries outside
 *                     [0, nkb) are ignored; kv_cnt is clamped to [0, cap]
 *   scale             logit scale, normally 1/sqrt(d)
 *   out               [B,H,Nq,d], fp32 (SA_OUT_F32) or bf16 (SA_OUT_BF16)
 *   err_flag          optional device int32, zero on entry. A CTA whose bounded
 *                     device wait gives up sets bits in it, drains its own copies
 *                     and MMAs, frees its tensor memory and exits; CTAs that start
 *                     after that find the flag set and skip their work. The call
 *                     itself still returns SA_OK (the kernel runs asynchronously):
 *                     a non-zero flag after the stream completes means
 *                     SA_ERR_TIMEOUT and the output is not valid. The flag is
 *                     sticky: clear it before the next call.
 * Ranges: probabilities enter the value products as fp16 at most 2^11 (relative to the
 * row's running maximum); with order 1 the operand scale * alpha * q_t is fp16 too, and
 * a row with |q| above 2^15 / (2^11 scale) (181 at d = 128) rescales its maximum earlier
 * so that the operand stays below 2^15. The pool's fp16 tables (V, value sums, M_j) are
 * checked by the pool (SA_FLAG_RANGE in its err_flag); given the same err_flag, a forward
 * that starts after a range error finds the flag set and skips its work.
 */
int sparse_attn_forward(const uint16_t* q, const uint16_t* k, const uint16_t* v16,
                        const uint16_t* kbar16, const uint16_t* vsum16, const uint16_t* M,
                        const int32_t* kv_idx, const int32_t* kv_cnt, int cap,
                        int B, int H, int Nq, int Nk, int d, int block, int order,
                        float scale, void* out, int out_dtype, int32_t* err_flag,
                        void* stream);

/*
 * The forward with the key blocks of every query tile shared out among `splits` CTAs
 * (whole runs of 64 blocks each), for grids too small to fill the GPU evenly: each CTA
 * runs the same online softmax over its own blocks (kept ones exactly, the others by
 * their compensation terms) and writes its unnormalised numerator with its running
 * maximum m_s (base 2) and denominator l_s; a second kernel merges the splits of every
 * row, o_t = sum_s 2^(m_s - M) N_s / sum_s 2^(m_s - M) l_s with M = max_s m_s. The
 * result equals sparse_attn_forward's up to fp32 rounding (the terms are summed in
 * another order). The pages describe one pass per query tile; the split is a scheduling
 * choice of this library.
 *   splits     1 <= splits <= SA_MAX_SPLITS; 1 is sparse_attn_forward (work may be NULL)
 *   work       device scratch owned by the caller, 16-byte aligned, at least
 *              sparse_attn_forward_work_bytes(B, H, Nq, d, splits) bytes:
 *              [splits][B*H][Nq][d] fp32 numerators, then [splits][B*H][Nq] (m, l) pairs
 *   others     as for sparse_attn_forward (same checks and the same err_flag contract)
 * Two launches when splits > 1 (forward, merge), one otherwise.
 */
int sparse_attn_forward_split(const uint16_t* q, const uint16_t* k, const uint16_t* v16,
                              const uint16_t* kbar16, const uint16_t* vsum16, const uint16_t* M,
                              const int32_t* kv_idx, const int32_t* kv_cnt, int cap, int B, int H,
                              int Nq, int Nk, int d, int block, int order, float scale, int splits,
                              float* work, void* out, int out_dtype, int32_t* err_flag,
                              void* stream);

/* Bytes of `work` sparse_attn_forward_split needs: splits * B * H * Nq * (d + 2) * 4 when
 * splits > 1, else 0. Host only. */
int sparse_attn_forward_work_bytes(int B, int H, int Nq, int d, int splits, size_t* bytes);

/*
 * Host-side choice of the split count for a problem shape: *splits = 1 unless splitting
 * shortens a model of the grid's schedule (CTAs of 1/S the work plus a fixed setup,
 * started in grid order on the first free SM of `sms`) by at least 3%; *work_bytes = the
 * scratch it needs. sms = 0 asks the current device for its SM count. No launch.
 */
int sparse_attn_forward_split_plan(int B, int H, int Nq, int Nk, int d, int block, int sms,
                                   int* splits, size_t* work_bytes);

/* Message for the last error returned on the calling thread ("" if none). */
const char* sparse_attn_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H_ */
