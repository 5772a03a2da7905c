// sol_reblock kernels: the adaptive partition of the keys and the row
// gathers / scatters around the unchanged Sol kernels.
//
// Spark-H3 news page, Spark-Reblock bullet: the fixed tiles are replaced by
// an adaptive partition; two rows are similar when their score patterns
// against the other side are, measured by the cosine under the Mahalanobis
// metric of the opposite side's second moment; a hierarchical splitter
// divides groups until every leaf has the block size.  The workflow
// paragraph fixes reblock_layout=q_reuse_k: queries take the keys' order.
//
// Reading (the same as the oracle's): per (b, h)
//   M  = mean of q q^T over the video query rows, + 1e-4 trace(M) / D * I;
//   y_t = normalise(k_t L), L the lower Cholesky factor of M, for the key rows
//        past the prefix blocks (which stay in place), so y.y' is the
//        Mahalanobis cosine;
//   a group of n > 64 rows splits along its principal axis (REBLOCK_ITERS
//        power steps on its covariance, started from its first row minus its
//        mean): the 64 * ceil(ceil(n / 64) / 2) rows of lowest projection
//        (ties to the lower row) go left, the rest right, each part keeping
//        ascending row order; so the partial leaf is last and every leaf
//        lists its rows ascending.
//
// Kernels, in launch order:
//   rb_moment_tc_kernel -- partial sums of q q^T over 2048-row chunks on the
//                        tensor cores (D = 128; rb_moment_kernel, fp32 FMAs,
//                        for D = 64);
//   rb_factor_kernel  -- one CTA per head: the partials summed in a fixed
//                        order, the ridge, the Cholesky factor in shared memory;
//   rb_whiten_tc_kernel -- y = normalise(k L) on the tensor cores, L split into
//                        three bf16 terms (D = 128; rb_whiten_kernel, fp32
//                        FMAs with L loaded once per 8 tiles, for D = 64), and
//                        the initial (identity) order;
//   per level of the hierarchy, for the levels whose groups hold at least
//   512 rows (D = 128):
//     rb_shift0_kernel -- (root only) a sample mean per head, the root's shift;
//     rb_gram_tc_kernel -- each group's shifted Gram matrix on the tensor cores
//                        (partials per CTA and group);
//     rb_axis_kernel  -- one CTA per group: the covariance from the partials,
//                        the power steps, the group's mean for the next level;
//     rb_split_kernel / rb_split_cluster_kernel with the axis given -- the
//                        projection pass, the select and the partition;
//   for the other levels, rb_split_kernel -- one CTA per group: mean, power
//                        steps and projections as 64-bit keys (order-
//                        preserving float bits, row index), the split rank
//                        found by a radix select, then a stable partition of
//                        the group's rows;
//   rb_perm_kernel    -- perm[pos] = original row at position pos;
//   gather / scatter  -- rows of a BTHD tensor into / out of a head-major
//                        [B, H, N, D] copy in the partition's order.
//
// Every reduction runs in a fixed order, so the partition is deterministic.
#include <math.h>

#include <cooperative_groups.h>

#include <atomic>

#include "common.cuh"
#include "ptx.cuh"   // packed f32x2 arithmetic

namespace sol {

namespace {

constexpr int kMomRows = 2048;       // query rows per partial-moment CTA
constexpr int kMomStage = 32;        // rows staged in shared memory at a time
constexpr int kSplitUnroll = 4;      // rows in flight per row slot

__host__ __device__ inline int rb_left(int n) { return kBlock * ((((n + kBlock - 1) / kBlock) + 1) / 2); }

// Group s of level lvl (its bits, most significant first, choose left / right
// at each level above): start and length in the video rows' order; false if
// an ancestor is already a leaf.
__device__ inline bool rb_segment(int n_v, int lvl, int s, int& start, int& len) {
  start = 0;
  len = n_v;
  for (int l = lvl - 1; l >= 0; --l) {
    if (len <= kBlock) return false;
    const int left = rb_left(len);
    if ((s >> l) & 1) { start += left; len -= left; } else { len = left; }
  }
  return true;
}

__device__ __forceinline__ float4 ld_bf16x4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
  const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}

// Partial second moment of the video query rows: grid (chunks, B*H).
template <int D>
__global__ void __launch_bounds__(256) rb_moment_kernel(const ReblockArgs a) {
  constexpr int TS = D / 16;   // each thread owns a TS x TS tile of the D x D moment
  __shared__ __align__(16) float xs[kMomStage][D];
  const int tid = threadIdx.x, ti = tid >> 4, tj = tid & 15;
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int r0 = a.q_lo + blockIdx.x * kMomRows, r1 = min(a.q_lo + a.n_q, r0 + kMomRows);
  const __nv_bfloat16* qb = a.q + (int64_t)b * a.sb + (int64_t)h * a.sh;
  uint64_t acc[TS][TS / 2];   // packed column pairs
#pragma unroll
  for (int i = 0; i < TS; ++i)
#pragma unroll
    for (int j = 0; j < TS / 2; ++j) acc[i][j] = 0ull;
  for (int s0 = r0; s0 < r1; s0 += kMomStage) {
    __syncthreads();
    for (int idx = tid; idx < kMomStage * (D / 4); idx += 256) {
      const int r = idx / (D / 4), c4 = (idx % (D / 4)) * 4, row = s0 + r;
      const float4 v = row < r1 ? ld_bf16x4(qb + (int64_t)row * a.sn + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(&xs[r][c4]) = v;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < kMomStage; ++r) {
      float u[TS];
      uint64_t w2[TS / 2];
#pragma unroll
      for (int i = 0; i < TS; i += 4) {
        const float4 x = *reinterpret_cast<const float4*>(&xs[r][ti * TS + i]);
        const float4 y = *reinterpret_cast<const float4*>(&xs[r][tj * TS + i]);
        u[i] = x.x; u[i + 1] = x.y; u[i + 2] = x.z; u[i + 3] = x.w;
        w2[i / 2] = f2pack(y.x, y.y);
        w2[i / 2 + 1] = f2pack(y.z, y.w);
      }
      // packed f32x2 FMAs over column pairs (each half an ordinary fp32 FMA)
#pragma unroll
      for (int i = 0; i < TS; ++i) {
        const uint64_t u2 = f2pack(u[i], u[i]);
#pragma unroll
        for (int j = 0; j < TS / 2; ++j) acc[i][j] = ffma2(u2, w2[j], acc[i][j]);
      }
    }
  }
  float* out = a.mpart + ((int64_t)bh * a.mchunks + blockIdx.x) * D * D;
#pragma unroll
  for (int i = 0; i < TS; ++i)
#pragma unroll
    for (int j = 0; j < TS / 2; ++j) {
      float lo, hi;
      f2unpack(acc[i][j], lo, hi);
      *reinterpret_cast<float2*>(&out[(ti * TS + i) * D + tj * TS + 2 * j]) = make_float2(lo, hi);
    }
}

// The same partial moments on the tensor cores (D = 128): grid (chunks, B*H),
// 128 threads.  The products of bf16 queries are exact and tcgen05 sums them
// in fp32, as the FMA kernel does (in another order).  Lane 0 of warp 0
// streams 64-row Q tiles (both 64-dim chunks, SW128) through a kMomStages
// ring; warp 1 issues M = N = D = 128, K = 16-row MMAs with A = Q^T and
// B = Q read MN-major from the same tile, accumulating the chunk's moment in
// TMEM; then every warp copies its 32 TMEM lanes (rows of the moment) out.
constexpr int kMomTcRows = 64;    // query rows per tile
constexpr int kMomStages = 4;     // tiles in flight
struct MomBars {
  uint64_t full[kMomStages], empty[kMomStages], done;
  uint32_t tmem;
  int abort_flag;
};
constexpr int kMomTile = kMomTcRows * 128 * 2;   // 16 KB: two 8 KB chunks of 64 dims
constexpr size_t kMomTcSmem = 1024 + kMomStages * kMomTile + sizeof(MomBars);

__global__ void __launch_bounds__(128) rb_moment_tc_kernel(const __grid_constant__ CUtensorMap mq, const ReblockArgs a) {
  constexpr int D = 128;
  extern __shared__ uint8_t mom_smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(mom_smem_raw) + 1023) & ~uintptr_t(1023));
  MomBars& bar = *reinterpret_cast<MomBars*>(ring + kMomStages * kMomTile);
  volatile int* abort_flag = &bar.abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int r0 = a.q_lo + blockIdx.x * kMomRows, r1 = min(a.q_lo + a.n_q, r0 + kMomRows);
  const int ntile = (r1 - r0 + kMomTcRows - 1) / kMomTcRows;   // >= 1; rows past N read as zeros
  if (tid == 0) {
    for (int s = 0; s < kMomStages; ++s) { mbar_init(&bar.full[s], 1); mbar_init(&bar.empty[s], 1); }
    mbar_init(&bar.done, 1);
    bar.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" :: "r"(smem_u32(&bar.tmem)), "r"(128));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncwarp();
  __syncthreads();
  fence_after();
  const uint32_t tmem = bar.tmem;
  if (warp == 0) {
    if (lane == 0) {   // TMA producer
      int nl = 0;
      for (int t = 0; t < ntile; ++t) {
        const int s = t % kMomStages, n = t / kMomStages;
        if (!wait_bar(&bar.empty[s], (n & 1) ^ 1, abort_flag, a.status)) break;
        mbar_expect_tx(&bar.full[s], kMomTile);
        ++nl;
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(ring + s * kMomTile + c * (kMomTile / 2), &mq, c * 64, h, r0 + kMomTcRows * t, b, &bar.full[s]);
      }
      for (int s = 0; s < kMomStages; ++s) {   // every armed load lands before the CTA may exit
        const int cnt = (nl + kMomStages - 1 - s) / kMomStages;
        if (cnt) drain_bar(&bar.full[s], (cnt - 1) & 1, a.status);
      }
    }
  } else if (warp == 1) {   // MMA issuer (the whole warp; one elected lane issues)
    constexpr uint32_t id = idesc_bf16(128, 128, 1, 1);   // A and B both MN-major (dims contiguous)
    bool ok = true;
    for (int t = 0; t < ntile && ok; ++t) {
      const int s = t % kMomStages, n = t / kMomStages;
      ok = __all_sync(0xffffffffu, wait_bar(&bar.full[s], n & 1, abort_flag, a.status));
      if (!ok) break;
      fence_after();
      // MN-major SW128: 64-dim chunks 8 KB apart (LBO), 8-row groups 1024 B apart (SBO); K = 16 rows = 2048 B
      const uint64_t dsc = sdesc(smem_u32(ring + s * kMomTile), kMomTile / 2, 1024);
#pragma unroll
      for (int kk = 0; kk < kMomTcRows / 16; ++kk)
        mma_ss_w(tmem, dsc + (uint64_t)(kk * 128), dsc + (uint64_t)(kk * 128), id, (t > 0 || kk > 0) ? 1u : 0u);
      mma_commit_w(&bar.empty[s]);   // the stage is free once these MMAs have read it
    }
    mma_commit_w(&bar.done);
  }
  // every warp: its 32 TMEM lanes = rows 32w .. 32w+31 of the moment, 128 columns each
  const bool ok = __all_sync(0xffffffffu, wait_bar(&bar.done, 0, abort_flag, a.status));
  fence_after();
  if (ok && !*abort_flag) {
    float* out = a.mpart + ((int64_t)bh * a.mchunks + blockIdx.x) * D * D + (int64_t)(32 * warp + lane) * D;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * warp) << 16);
    for (int c = 0; c < D / 32; ++c) {
      float v[32];
      tmem_ld32(lane_addr + 32 * c, v);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(out + 32 * c + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
    }
  }
  fence_before();
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(128));
  }
}

// M = (sum of the partials, chunk order) / n_q + ridge; its lower Cholesky
// factor L (left-looking, one column at a time): one CTA per (b, h).
template <int D>
__global__ void __launch_bounds__(256) rb_factor_kernel(const ReblockArgs a) {
  constexpr int LD = D + 1;                    // padded rows: column reads hit distinct banks
  extern __shared__ __align__(16) float M[];   // [D][LD]
  __shared__ float s_ridge;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, bh = blockIdx.x;
  const float* part = a.mpart + (int64_t)bh * a.mchunks * D * D;
  const float inv_n = 1.f / (float)a.n_q;
  {   // thread tid sums float4 f = tid + 256 k of every chunk's partial, all k's loads in flight
    constexpr int KF = D * D / 4 / 256;
    float4 acc[KF];
#pragma unroll
    for (int k = 0; k < KF; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < a.mchunks; ++c) {
      const float4* src = reinterpret_cast<const float4*>(part + (int64_t)c * D * D);
#pragma unroll
      for (int k = 0; k < KF; ++k) {
        const float4 v = src[tid + 256 * k];
        acc[k].x += v.x; acc[k].y += v.y; acc[k].z += v.z; acc[k].w += v.w;
      }
    }
#pragma unroll
    for (int k = 0; k < KF; ++k) {
      const int idx = 4 * (tid + 256 * k), i = idx / D, j = idx % D;
      M[i * LD + j] = acc[k].x * inv_n;
      M[i * LD + j + 1] = acc[k].y * inv_n;
      M[i * LD + j + 2] = acc[k].z * inv_n;
      M[i * LD + j + 3] = acc[k].w * inv_n;
    }
  }
  __syncthreads();
  if (warp == 0) {
    float t = 0.f;
    for (int i = lane; i < D; i += 32) t += M[i * LD + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) s_ridge = t > 0.f ? 1e-4f * t / (float)D : 1.f;
  }
  __syncthreads();
  if (tid < D) M[tid * LD + tid] += s_ridge;
  __syncthreads();
  for (int j = 0; j < D; ++j) {
    if (warp == 0) {   // diagonal: M[j][j] - sum_c<j L[j][c]^2, lanes strided, fixed-order tree
      float t = 0.f;
      for (int c = lane; c < j; c += 32) t = fmaf(M[j * LD + c], M[j * LD + c], t);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) {
        float d = M[j * LD + j] - t;
        if (!(d > 0.f)) d = s_ridge;   // cannot happen with the ridge; keeps L finite
        M[j * LD + j] = sqrtf(d);
      }
    }
    __syncthreads();
    const float ljj = M[j * LD + j];
    for (int i = j + 1 + tid; i < D; i += 256) {
      // sum_c<j L[i][c] L[j][c] in four interleaved partial sums (c mod 4), then added in order
      float t0 = 0.f, t1 = 0.f, t2 = 0.f, t3 = 0.f;
      const float* Li = M + i * LD;
      const float* Lj = M + j * LD;
      int c = 0;
      for (; c + 4 <= j; c += 4) {
        t0 = fmaf(Li[c], Lj[c], t0);
        t1 = fmaf(Li[c + 1], Lj[c + 1], t1);
        t2 = fmaf(Li[c + 2], Lj[c + 2], t2);
        t3 = fmaf(Li[c + 3], Lj[c + 3], t3);
      }
      for (; c < j; ++c) t0 = fmaf(Li[c], Lj[c], t0);
      M[i * LD + j] = (M[i * LD + j] - ((t0 + t1) + (t2 + t3))) / ljj;
    }
    __syncthreads();
  }
  float* L = a.L + (int64_t)bh * D * D;
  for (int idx = tid; idx < D * D; idx += 256) L[idx] = (idx % D) <= (idx / D) ? M[(idx / D) * LD + idx % D] : 0.f;
}

// y = normalise(k L) for the video key rows: grid (ceil(n_v / (64 kWhTiles)), B*H).
// A CTA loads L (D x D fp32) into shared memory once and whitens kWhTiles
// tiles of 64 rows.  Warp w owns the 16 columns 16w .. 16w+15 of y, lane the
// rows lane and lane+32 of the tile; L is lower triangular, so column j
// gathers only i >= j and warp w's dot products start at i = 16w (the
// skipped terms are exact zeros: the sums are those of the full loop).
constexpr int kWhTiles = 8;
template <int D>
__global__ void __launch_bounds__(256) rb_whiten_kernel(const ReblockArgs a) {
  constexpr int LK = D + 1;   // padded key rows: lanes read rows lane, lane+32 on distinct banks
  constexpr int CPW = D / 8;  // columns per warp
  extern __shared__ __align__(16) float sm[];
  float* Ls = sm;                     // [D][D]
  float* ks = sm + D * D;             // [64][LK]
  float* ssq = ks + kBlock * LK;      // [8][64] partial squared norms
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const float* Lg = a.L + (int64_t)bh * D * D;
  for (int idx = tid * 4; idx < D * D; idx += 256 * 4)
    *reinterpret_cast<float4*>(&Ls[idx]) = *reinterpret_cast<const float4*>(&Lg[idx]);
  const __nv_bfloat16* kb = a.k + (int64_t)b * a.sb + (int64_t)h * a.sh;
  const int c0 = CPW * warp;
  for (int it = 0; it < kWhTiles; ++it) {
    const int t0 = (blockIdx.x * kWhTiles + it) * kBlock;
    if (t0 >= a.n_v) break;   // uniform over the CTA
    __syncthreads();          // the previous tile's ks and ssq are consumed (and L has landed)
    for (int idx = tid; idx < kBlock * (D / 4); idx += 256) {
      const int r = idx / (D / 4), c4 = (idx % (D / 4)) * 4, t = t0 + r;
      const float4 v = t < a.n_v ? ld_bf16x4(kb + (int64_t)(a.n_fix + t) * a.sn + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
      float* dst = &ks[r * LK + c4];
      dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
    }
    __syncthreads();
    uint64_t y2[2][CPW / 2];   // rows lane, lane+32; packed column pairs
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int c = 0; c < CPW / 2; ++c) y2[r][c] = 0ull;
    for (int i = c0; i < D; ++i) {
      uint64_t l2[CPW / 2];
#pragma unroll
      for (int c = 0; c < CPW; c += 4) {   // broadcast: the whole warp reads the same columns
        const float4 l4 = *reinterpret_cast<const float4*>(&Ls[i * D + c0 + c]);
        l2[c / 2] = f2pack(l4.x, l4.y);
        l2[c / 2 + 1] = f2pack(l4.z, l4.w);
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float kv = ks[(lane + 32 * r) * LK + i];
        const uint64_t k2 = f2pack(kv, kv);
#pragma unroll
        for (int c = 0; c < CPW / 2; ++c) y2[r][c] = ffma2(k2, l2[c], y2[r][c]);
      }
    }
    float y[2][CPW];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < CPW / 2; ++c) {
        f2unpack(y2[r][c], y[r][2 * c], y[r][2 * c + 1]);
        ss = fmaf(y[r][2 * c], y[r][2 * c], ss);
        ss = fmaf(y[r][2 * c + 1], y[r][2 * c + 1], ss);
      }
      ssq[warp * kBlock + lane + 32 * r] = ss;
    }
    __syncthreads();
    float* Yg = a.Y + ((int64_t)bh * a.n_v + t0) * D;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = lane + 32 * r;
      float ss = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2) ss += ssq[w2 * kBlock + row];   // fixed order over the column groups
      const float inv = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
      if (t0 + row < a.n_v) {
        float* dst = Yg + (int64_t)row * D + c0;
#pragma unroll
        for (int c = 0; c < CPW; c += 4)
          *reinterpret_cast<float4*>(dst + c) =
              make_float4(y[r][c] * inv, y[r][c + 1] * inv, y[r][c + 2] * inv, y[r][c + 3] * inv);
      }
    }
    if (tid < kBlock && t0 + tid < a.n_v) a.ord[(int64_t)bh * a.n_v + t0 + tid] = t0 + tid;
  }
}

// y = normalise(k L) on the tensor cores (D = 128).  L (fp32) is split into three
// bf16 terms L = L1 + L2 + L3 (each the rounding of what the previous ones leave,
// 2^-24 of L in all), laid out MN-major in shared memory; every 128-row key tile
// is A (K-major, from TMA) and the three products accumulate in TMEM in fp32: the
// products are exact and the split is as fine as fp32's own rounding.
// Persistent: grid min(148, tiles), the tiles of all heads (head-major) split
// evenly over the CTAs; a CTA converts L again where its range enters a new head.
// Warp 4 streams the key tiles through a kWhTcStages ring, warp 5 issues the 24
// MMAs of a tile into one of two TMEM accumulators, and warps 0-3 (warp w: TMEM
// lanes 32w .. 32w+31) take each row's norm and write the unit vector while the
// MMAs of the next tile fill the other accumulator.
constexpr int kWhTcRows = 128;
constexpr int kWhTcCtas = 148;
constexpr int kWhTcThreads = 192;
constexpr int kWhTcStages = 3;
struct WhBars {
  uint64_t full[kWhTcStages], empty[kWhTcStages], acc_full[2], acc_free[2], done;
  uint32_t tmem;
  int abort_flag;
};
constexpr int kWhTile = kWhTcRows * 128 * 2;     // 32 KB: a K tile, or one bf16 term of L
constexpr int kWhStw = 4 * 32 * 33 * 4;          // the epilogue warps' row transposes (padded)
constexpr size_t kWhTcSmem = 1024 + (3 + kWhTcStages) * kWhTile + kWhStw + sizeof(WhBars);
static_assert(kWhTcSmem <= 232448, "whitening kernel shared memory");

// grid ceil(tiles / chunk), kWhTcThreads threads; tph = 128-row tiles per head
__global__ void __launch_bounds__(kWhTcThreads, 1) rb_whiten_tc_kernel(const __grid_constant__ CUtensorMap mk,
                                                                        const ReblockArgs a, int tph, int chunk) {
  constexpr int D = 128;
  extern __shared__ uint8_t wh_smem_raw[];
  uint8_t* Lt = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(wh_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = Lt + 3 * kWhTile;
  float* stw = reinterpret_cast<float*>(ring + kWhTcStages * kWhTile);   // [4][32][33]
  WhBars& bar = *reinterpret_cast<WhBars*>(reinterpret_cast<uint8_t*>(stw) + kWhStw);
  volatile int* abort_flag = &bar.abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int TT = a.B * a.H * tph;
  const int t0 = blockIdx.x * chunk, t1 = min(TT, t0 + chunk);
  if (tid == 0) {
    for (int s = 0; s < kWhTcStages; ++s) { mbar_init(&bar.full[s], 1); mbar_init(&bar.empty[s], 1); }
    for (int b2 = 0; b2 < 2; ++b2) { mbar_init(&bar.acc_full[b2], 1); mbar_init(&bar.acc_free[b2], 4); }
    mbar_init(&bar.done, 1);
    bar.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" :: "r"(smem_u32(&bar.tmem)), "r"(256));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncwarp();
  __syncthreads();
  fence_after();
  const uint32_t tmem = bar.tmem;
  int q = 0;   // tiles of this CTA so far (uniform)
  bool ok = true, mma_issued = false;
  for (int T = t0; T < t1 && ok;) {   // one segment: the range's tiles of one head
    const int bh = T / tph, b = bh / a.H, h = bh % a.H;
    const int Te = min(t1, (bh + 1) * tph), ntile = Te - T, k0 = T - bh * tph;
    // L's three bf16 terms, MN-major SW128: element (i, j) in chunk j/64, row i, 16-byte unit
    // (j%64)/8 at position unit ^ (i & 7); thread tid converts units tid, tid+192, ... (8 columns each)
    const float* Lg = a.L + (int64_t)bh * D * D;
    for (int u = tid; u < D * D / 8; u += kWhTcThreads) {
      const int i = u / (D / 8), j0 = (u % (D / 8)) * 8;
      const float4 x0 = *reinterpret_cast<const float4*>(Lg + i * D + j0);
      const float4 x1 = *reinterpret_cast<const float4*>(Lg + i * D + j0 + 4);
      const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      uint32_t w1[4], w2[4], w3[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        float r0 = x[e], r1 = x[e + 1];
        const __nv_bfloat162 h1 = __floats2bfloat162_rn(r0, r1);
        r0 -= __low2float(h1); r1 -= __high2float(h1);
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(r0, r1);
        r0 -= __low2float(h2); r1 -= __high2float(h2);
        const __nv_bfloat162 h3 = __floats2bfloat162_rn(r0, r1);
        w1[e / 2] = *reinterpret_cast<const uint32_t*>(&h1);
        w2[e / 2] = *reinterpret_cast<const uint32_t*>(&h2);
        w3[e / 2] = *reinterpret_cast<const uint32_t*>(&h3);
      }
      const int off = (j0 / 64) * (kWhTile / 2) + i * 128 + ((((j0 % 64) / 8) ^ (i & 7)) << 4);
      *reinterpret_cast<uint4*>(Lt + off) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
      *reinterpret_cast<uint4*>(Lt + kWhTile + off) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
      *reinterpret_cast<uint4*>(Lt + 2 * kWhTile + off) = make_uint4(w3[0], w3[1], w3[2], w3[3]);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the terms feed the tensor cores
    __syncthreads();
    if (warp == 4) {   // TMA producer: 128-row key tiles (two 64-dim chunks)
      if (lane == 0) {
        int nl = 0;
        for (int t = 0; t < ntile; ++t) {
          const int g = q + t, s = g % kWhTcStages, n = g / kWhTcStages;
          if (!wait_bar(&bar.empty[s], (n & 1) ^ 1, abort_flag, a.status)) break;
          mbar_expect_tx(&bar.full[s], kWhTile);
          ++nl;
          const int row = a.n_fix + (k0 + t) * kWhTcRows;
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(ring + s * kWhTile + c * (kWhTile / 2), &mk, c * 64, h, row, b, &bar.full[s]);
        }
        if (nl < ntile) {   // after an abort: every armed load lands before the CTA moves on
          for (int t = max(0, nl - kWhTcStages); t < nl; ++t) {   // each stage's last load
            const int g = q + t;
            drain_bar(&bar.full[g % kWhTcStages], (g / kWhTcStages) & 1, a.status);
          }
        }
      }
      __syncwarp();
    } else if (warp == 5) {   // MMA issuer
      constexpr uint32_t id = idesc_bf16(128, 128, 0, 1);   // A = keys K-major, B = L terms MN-major
      const uint64_t ldsc0 = sdesc(smem_u32(Lt), kWhTile / 2, 1024);
      for (int t = 0; t < ntile; ++t) {
        const int g = q + t, s = g % kWhTcStages, n = g / kWhTcStages, bb = g & 1, u = g >> 1;
        // tile g's keys have landed, and accumulator bb's previous tile (g - 2) has been read
        if (!__all_sync(0xffffffffu, wait_bar(&bar.full[s], n & 1, abort_flag, a.status) &&
                                         wait_bar(&bar.acc_free[bb], (u & 1) ^ 1, abort_flag, a.status)))
          break;
        fence_after();
        const uint64_t adsc = sdesc(smem_u32(ring + s * kWhTile), 16, 1024);
        const uint32_t acc = tmem + 128 * bb;
#pragma unroll
        for (int term = 0; term < 3; ++term) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t aoff = (uint64_t)(((kk >> 2) * (kWhTile / 2) + (kk & 3) * 32) >> 4);
            const uint64_t boff = (uint64_t)((term * kWhTile + kk * 2048) >> 4);
            mma_ss_w(acc, adsc + aoff, ldsc0 + boff, id, (term > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_issued = true;
        mma_commit_w(&bar.empty[s]);
        mma_commit_w(&bar.acc_full[bb]);
      }
    } else {   // warps 0-3: row 32 warp + lane of each tile from TMEM: its norm, then the unit vector
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * warp) << 16);
      for (int t = 0; t < ntile; ++t) {
        const int g = q + t, bb = g & 1, u = g >> 1;
        if (!__all_sync(0xffffffffu, wait_bar(&bar.acc_full[bb], u & 1, abort_flag, a.status))) break;
        fence_after();
        const int row = (k0 + t) * kWhTcRows + 32 * warp + lane;   // position among the video rows
        float ss = 0.f;
        for (int c = 0; c < D / 32; ++c) {
          float v[32];
          tmem_ld32(lane_addr + 128 * bb + 32 * c, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ss = fmaf(v[e], v[e], ss);
        }
        const float inv = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
        // second read of the row: the unit vector, 32 columns at a time, turned through shared
        // memory so that each store writes four whole 128-byte row pieces
        float* sw = stw + warp * 32 * 33;
        const int row0 = (k0 + t) * kWhTcRows + 32 * warp;   // the warp's first row
        for (int c = 0; c < D / 32; ++c) {
          float v[32];
          tmem_ld32(lane_addr + 128 * bb + 32 * c, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) sw[lane * 33 + e] = v[e] * inv;
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {   // rows 4k + lane / 8, columns 32c + 4 (lane % 8) .. + 3
            const int r = 4 * k + (lane >> 3), cc = 4 * (lane & 7);
            if (row0 + r < a.n_v)
              *reinterpret_cast<float4*>(a.Y + ((int64_t)bh * a.n_v + row0 + r) * D + 32 * c + cc) =
                  make_float4(sw[r * 33 + cc], sw[r * 33 + cc + 1], sw[r * 33 + cc + 2], sw[r * 33 + cc + 3]);
          }
          __syncwarp();
        }
        if (row < a.n_v) a.ord[(int64_t)bh * a.n_v + row] = row;
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.acc_free[bb]);   // this warp has read tile g's accumulator
      }
    }
    q += ntile;
    T = Te;
    fence_before();
    ok = !__syncthreads_or(*abort_flag);   // every MMA of the segment has been read: L may change
    fence_after();
  }
  fence_before();
  __syncthreads();
  if (warp == 5) {
    // every issued MMA has landed before TMEM is released (after an abort the
    // epilogue may not have waited for the last ones)
    if (mma_issued) {
      mma_commit_w(&bar.done);
      drain_bar(&bar.done, 0, a.status);
    }
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(256));
  }
}

// Sum of a per-lane float4 over the CTA's row slots into out[D] (fixed order).
template <int D, int W>
__device__ __forceinline__ void rb_block_sum(float4 v, float4 (*red)[D / 4], float* out, float scale) {
  constexpr int LPR = D / 4, RPW = 32 / LPR;   // lanes per row, rows per warp
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (RPW == 2) {
    v.x += __shfl_xor_sync(0xffffffffu, v.x, 16);
    v.y += __shfl_xor_sync(0xffffffffu, v.y, 16);
    v.z += __shfl_xor_sync(0xffffffffu, v.z, 16);
    v.w += __shfl_xor_sync(0xffffffffu, v.w, 16);
  }
  if (lane < LPR) red[warp][lane] = v;
  __syncthreads();
  if (threadIdx.x < LPR) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int w = 0; w < W; ++w) {
      const float4 t = red[w][threadIdx.x];
      s.x += t.x; s.y += t.y; s.z += t.z; s.w += t.w;
    }
    out[4 * threadIdx.x + 0] = s.x * scale;
    out[4 * threadIdx.x + 1] = s.y * scale;
    out[4 * threadIdx.x + 2] = s.z * scale;
    out[4 * threadIdx.x + 3] = s.w * scale;
  }
  __syncthreads();
}

// Dot product of a row's lane quad with x over the row's lanes (all of them get it).
template <int D>
__device__ __forceinline__ float rb_row_dot(float4 y, float4 x) {
  float t = y.x * x.x;
  t = fmaf(y.y, x.y, t);
  t = fmaf(y.z, x.z, t);
  t = fmaf(y.w, x.w, t);
#pragma unroll
  for (int o = D / 8; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}

__device__ __forceinline__ float rb_norm(const float* v, int D, float* s_tmp) {
  // single-warp fixed-order norm of v[D], broadcast through shared memory
  if (threadIdx.x < 32) {
    float t = 0.f;
    for (int i = threadIdx.x; i < D; i += 32) t = fmaf(v[i], v[i], t);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (threadIdx.x == 0) *s_tmp = sqrtf(t);
  }
  __syncthreads();
  const float n = *s_tmp;
  __syncthreads();
  return n;
}

__device__ inline size_t reblock_axis_floats_dev(const ReblockArgs& a) {
  return a.gram_levels == 0 ? 0 : ((size_t)(a.B * a.H) << (a.gram_levels - 1)) * 128;
}

// The group of level lvl that holds position pos: its index s among the level's
// 2^lvl groups (bits as in rb_segment), start and length; false if an ancestor is
// already a leaf.
__device__ inline bool rb_group_at(int n_v, int lvl, int pos, int& s, int& start, int& len) {
  s = 0;
  start = 0;
  len = n_v;
  for (int l = 0; l < lvl; ++l) {
    if (len <= kBlock) return false;
    const int left = rb_left(len);
    if (pos < start + left) {
      s = 2 * s;
      len = left;
    } else {
      s = 2 * s + 1;
      start += left;
      len -= left;
    }
  }
  return true;
}

// Split axes of the large groups from Gram matrices (D = 128).
//
// The power steps z = C w, C = sum over the group of (y - mean)(y - mean)^T,
// need C only, so a group's C is built once instead of streaming its rows
// once per step.  With a shift c and x = y - c,
//   G = sum x x^T,  s1 = sum x,  C = G - s1 s1^T / n,  mean = c + s1 / n.
// The subtraction cancels |mean - c|^2 against C's spread, so c has to lie near
// the mean: it is the parent group's mean (computed the same way one level up),
// and for the root the mean of 1,024 evenly spaced rows (rb_shift0_kernel).
// (The whitened unit keys of a head are close to isotropic: shifting by one row
// instead, |mean - c|^2 is about 100 times C's largest eigenvalue.)
// rb_gram_tc_kernel sums G on the tensor cores: each x (fp32) is split into
// two bf16 terms h + m (round to nearest each; the rest, below 2^-17 |x|, is
// dropped), and G = H^T H + H^T M + M^T H.  The dropped rest is a zero-mean
// rounding residual, so its share of G shrinks with the number of rows; the
// dropped M^T M is below 2^-18 of H^T H and sits mostly on the diagonal.  TMEM accumulates four tiles (256 rows, 16 K steps)
// at a time; four epilogue warps add each finished chunk into a running fp32
// sum (round to nearest) while the MMAs fill the other chunk buffer, so no
// accumulation in the tensor pipe runs longer than 16 steps.  The level's rows
// are cut into 64-row tiles (tiles never straddle a group: group starts are
// multiples of 64), the tiles of all heads split evenly over kGrCtas CTAs; each
// CTA flushes one partial (G, s1) per group it touches into slot (group index +
// CTA index), which is unique.  rb_axis_kernel sums a group's partials in CTA
// order, forms C, runs the power steps from r - mean (r the group's first row)
// and records the group's mean for the next level.
constexpr int kGramMinRows = 512;    // levels whose groups have at least this many rows
constexpr int kGrCtas = 148;
constexpr int kGrRows = 64;          // rows per tile: four K = 16 steps
constexpr int kGrChunk = 4;          // tiles per TMEM chunk
#ifndef SOL_GR_SLOTS
#define SOL_GR_SLOTS 3
#endif
#ifndef SOL_GR_STAGES
#define SOL_GR_STAGES 4
#endif
constexpr int kGrSlots = SOL_GR_SLOTS;     // fp32 staging slots per row: kGrSlots - 1 tiles in flight
constexpr int kGrStages = SOL_GR_STAGES;   // bf16 term stages between the converting warps and the MMAs
constexpr int kGrWarps = 16;         // converting warps 0-15; warp 16 issues the MMAs; 17-20 add the chunks
constexpr int kGrMmaWarp = kGrWarps;
constexpr int kGrThreads = 32 * (kGrWarps + 5);
constexpr int kGrRowsPerWarp = kGrRows / kGrWarps;
constexpr int kGrTerm = kGrRows * 128 * 2;         // 16 KB: one bf16 term, two 8 KB chunks of 64 dims
constexpr int kGrStage = 2 * kGrTerm;              // the two terms of a tile
constexpr int kGrStaging = kGrRows * 128 * 4;      // 32 KB: one fp32 tile
constexpr int kGramPartFloats = 128 * 128 + 128;   // G, then s1
struct GrBars {
  uint64_t full[kGrStages], empty[kGrStages], accf[2], accr[2], done;
  uint32_t tmem;
  int abort_flag;
};
constexpr size_t kGrSmem = 1024 + kGrStages * kGrStage + kGrSlots * kGrStaging + sizeof(GrBars);
static_assert(kGrSmem <= 232448, "Gram kernel shared memory");

// Means of level lvl's groups go to half (lvl + 1) & 1 of cbuf; the shifts of level
// lvl are read from half lvl & 1: the parent's mean, or the root's sample mean.
__device__ inline int64_t rb_shift_index(const ReblockArgs& a, int lvl, int bh, int s) {
  const int64_t half = (int64_t)reblock_axis_floats_dev(a) * (lvl & 1);
  return half / 128 + (lvl == 0 ? (int64_t)bh : ((int64_t)bh << (lvl - 1)) + (s >> 1));
}

// The root's shift: per head, the mean of min(n_v, 1024) evenly spaced rows;
// grid B*H, 1024 threads: sample i goes to warp i % 32, whose lanes hold four
// dimensions each; the 32 warp sums are added in warp order.
__global__ void __launch_bounds__(1024) rb_shift0_kernel(const ReblockArgs a) {
  constexpr int D = 128;
  __shared__ __align__(16) float4 part[32][D / 4];
  const int bh = blockIdx.x, S = min(a.n_v, 1024), warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* Yh = a.Y + (int64_t)bh * a.n_v * D;
  float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int i = warp; i < S; i += 32) {
    const float4 y = *reinterpret_cast<const float4*>(Yh + ((int64_t)i * a.n_v / S) * D + 4 * lane);
    t.x += y.x; t.y += y.y; t.z += y.z; t.w += y.w;
  }
  part[warp][lane] = t;
  __syncthreads();
  if (threadIdx.x < D) {
    float u = 0.f;
    for (int w = 0; w < 32; ++w) u += reinterpret_cast<const float*>(part[w])[threadIdx.x];
    a.cbuf[rb_shift_index(a, 0, bh, 0) * D + threadIdx.x] = u / (float)S;
  }
}

// grid ceil(tiles / chunk), kGrThreads threads; tph = 64-row tiles per head.
// TMEM columns: chunk buffers 0-127 and 128-255, the running sum 256-383.
__global__ void __launch_bounds__(kGrThreads, 1) rb_gram_tc_kernel(const ReblockArgs a, int lvl, int tph, int chunk) {
  constexpr int D = 128;
  extern __shared__ uint8_t gr_smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gr_smem_raw) + 1023) & ~uintptr_t(1023));
  float* stg = reinterpret_cast<float*>(ring + kGrStages * kGrStage);   // [kGrSlots][kGrRows][D]
  GrBars& bar = *reinterpret_cast<GrBars*>(stg + kGrSlots * kGrRows * D);
  // a converting warp's s1 goes to the first of its own staging rows once its copies are done
  auto s1_row = [&](int w) { return stg + w * kGrRowsPerWarp * D; };
  volatile int* abort_flag = &bar.abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int TT = a.B * a.H * tph;
  const int t0 = blockIdx.x * chunk, t1 = min(TT, t0 + chunk);
  if (tid == 0) {
    for (int b = 0; b < kGrStages; ++b) {
      mbar_init(&bar.full[b], kGrWarps);
      mbar_init(&bar.empty[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.accf[b], 1);
      mbar_init(&bar.accr[b], 4);
    }
    mbar_init(&bar.done, 1);
    bar.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kGrMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" :: "r"(smem_u32(&bar.tmem)), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncwarp();
  __syncthreads();
  fence_after();
  const uint32_t tmem = bar.tmem;
  int q = 0;    // tiles through the ring so far (uniform)
  int cc = 0;   // TMEM chunks so far (uniform)
  bool ok = true, mma_issued = false;
  for (int T = t0; T < t1 && ok;) {
    const int bh = T / tph, k0 = T % tph;
    int s, start, len;
    const bool live = rb_group_at(a.n_v, lvl, k0 * kGrRows, s, start, len) && len > kBlock;
    // a group that is a leaf here (or lies under one) is one tile: its start is a multiple of 64
    const int Te = live ? min(t1, bh * tph + (start + len + kGrRows - 1) / kGrRows) : T + 1;
    if (!live) {
      T = Te;
      continue;
    }
    const int ntile = Te - T, nchunk = (ntile + kGrChunk - 1) / kGrChunk;
    const int p_lo = k0 * kGrRows, p_hi = min(start + len, (Te - bh * tph) * kGrRows);
    const int32_t* ordh = a.ord + (int64_t)bh * a.n_v;
    const float* Yh = a.Y + (int64_t)bh * a.n_v * D;
    float* P = a.gpart + (size_t)(((int64_t)bh << lvl) + s + blockIdx.x) * kGramPartFloats;
    if (warp < kGrWarps) {   // staging copies, the shift and the bf16 split into the ring
      const float4 rv = *reinterpret_cast<const float4*>(a.cbuf + rb_shift_index(a, lvl, bh, s) * D + 4 * lane);
      float4 s1 = make_float4(0.f, 0.f, 0.f, 0.f);
      struct Ids { int v[kGrRowsPerWarp]; };
      auto ids_of = [&](int t) {
        Ids id;
#pragma unroll
        for (int j = 0; j < kGrRowsPerWarp; ++j) {
          const int pos = p_lo + t * kGrRows + warp * kGrRowsPerWarp + j;
          id.v[j] = (t < ntile && pos < p_hi) ? ordh[pos] : -1;
        }
        return id;
      };
      auto issue = [&](int t, const Ids id) {   // always one commit group, possibly empty
        float* dst = stg + ((t % kGrSlots) * kGrRows + warp * kGrRowsPerWarp) * D + 4 * lane;
#pragma unroll
        for (int j = 0; j < kGrRowsPerWarp; ++j)
          if (id.v[j] >= 0) cp_async16(dst + j * D, Yh + (int64_t)id.v[j] * D + 4 * lane);
        cp_async_commit();
      };
#pragma unroll
      for (int t = 0; t < kGrSlots - 1; ++t) issue(t, ids_of(t));
      Ids idn = ids_of(kGrSlots - 1);
      for (int t = 0; t < ntile; ++t) {
        issue(t + kGrSlots - 1, idn);   // empty past the segment's end
        idn = ids_of(t + kGrSlots);     // consumed by the next iteration's issue
        cp_async_wait<kGrSlots - 1>();  // this thread's copies of tile t have landed
        const int st = (q + t) % kGrStages, n = (q + t) / kGrStages;
        if (!__all_sync(0xffffffffu, wait_bar(&bar.empty[st], (n & 1) ^ 1, abort_flag, a.status))) break;
        const float* sp = stg + ((t % kGrSlots) * kGrRows + warp * kGrRowsPerWarp) * D + 4 * lane;
        uint8_t* base = ring + st * kGrStage;
#pragma unroll
        for (int j = 0; j < kGrRowsPerWarp; ++j) {
          const int R = warp * kGrRowsPerWarp + j;
          float x[4] = {0.f, 0.f, 0.f, 0.f};
          if (p_lo + t * kGrRows + R < p_hi) {
            const float4 y = *reinterpret_cast<const float4*>(sp + j * D);
            x[0] = y.x - rv.x; x[1] = y.y - rv.y; x[2] = y.z - rv.z; x[3] = y.w - rv.w;
            s1.x += x[0]; s1.y += x[1]; s1.z += x[2]; s1.w += x[3];
          }
          uint32_t th[2], tm[2];
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const __nv_bfloat162 h1 = __floats2bfloat162_rn(x[e], x[e + 1]);
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(x[e] - __low2float(h1), x[e + 1] - __high2float(h1));
            th[e / 2] = *reinterpret_cast<const uint32_t*>(&h1);
            tm[e / 2] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          // MN-major SW128: dims 4 lane .. 4 lane + 3 are chunk lane / 16, 16-byte unit (lane % 16) / 2
          // at position unit ^ (R & 7), half lane % 2
          const int off = (lane >> 4) * (kGrTerm / 2) + R * 128 + ((((lane & 15) >> 1) ^ (R & 7)) << 4) + ((lane & 1) << 3);
          *reinterpret_cast<uint2*>(base + off) = make_uint2(th[0], th[1]);
          *reinterpret_cast<uint2*>(base + kGrTerm + off) = make_uint2(tm[0], tm[1]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the terms feed the tensor cores
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.full[st]);
      }
      cp_async_wait<0>();
      *reinterpret_cast<float4*>(s1_row(warp) + 4 * lane) = s1;
    } else if (warp == kGrMmaWarp) {   // M = N = 128 (dims), K = 16 rows, A and B MN-major from the ring
      constexpr uint32_t id = idesc_bf16(128, 128, 1, 1);
      for (int t = 0; t < ntile; ++t) {
        const int kc = cc + t / kGrChunk, b = kc & 1, u = kc >> 1;
        const bool first = t % kGrChunk == 0, last = t % kGrChunk == kGrChunk - 1 || t == ntile - 1;
        // chunk buffer b is free once the epilogue has added its previous chunk
        if (first && !__all_sync(0xffffffffu, wait_bar(&bar.accr[b], (u & 1) ^ 1, abort_flag, a.status))) break;
        const int st = (q + t) % kGrStages, n = (q + t) / kGrStages;
        if (!__all_sync(0xffffffffu, wait_bar(&bar.full[st], n & 1, abort_flag, a.status))) break;
        fence_after();
        const uint64_t dH = sdesc(smem_u32(ring + st * kGrStage), kGrTerm / 2, 1024);
        const uint64_t dM = dH + (uint64_t)(kGrTerm >> 4);
        const uint32_t acc_addr = tmem + 128 * b;
#pragma unroll
        for (int kk = 0; kk < kGrRows / 16; ++kk) {
          const uint64_t o = (uint64_t)(kk * 128);   // 16 rows = 2048 bytes
          mma_ss_w(acc_addr, dH + o, dH + o, id, (!first || kk > 0) ? 1u : 0u);
          mma_ss_w(acc_addr, dH + o, dM + o, id, 1u);
          mma_ss_w(acc_addr, dM + o, dH + o, id, 1u);
        }
        mma_issued = true;
        mma_commit_w(&bar.empty[st]);
        if (last) mma_commit_w(&bar.accf[b]);
      }
    } else {   // warps 17-20: TMEM lanes 32 (warp % 4) + lane, i.e. row i of the chunk and of the sum
      const int i = 32 * (warp & 3) + lane;
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
      bool got = true;
      for (int c = 0; c < nchunk && got; ++c) {
        const int kc = cc + c, b = kc & 1, u = kc >> 1;
        got = __all_sync(0xffffffffu, wait_bar(&bar.accf[b], u & 1, abort_flag, a.status));
        if (!got) break;
        fence_after();
#pragma unroll 1
        for (int g = 0; g < D / 16; ++g) {   // sum (+)= chunk, 16 columns at a time
          float v[16], w2[16];
          tmem_ld16(lane_addr + 128 * b + 16 * g, v);
          if (c > 0) tmem_ld16(lane_addr + 256 + 16 * g, w2);
          tmem_wait_ld();
          if (c > 0) {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] += w2[e];
          }
          tmem_st16(lane_addr + 256 + 16 * g, reinterpret_cast<const uint32_t*>(v));
        }
        tmem_wait_st();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.accr[b]);
      }
      if (got) {   // row i of the segment's G
#pragma unroll 1
        for (int g = 0; g < D / 32; ++g) {
          float v[32];
          tmem_ld32(lane_addr + 256 + 32 * g, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(P + i * D + 32 * g + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
    }
    __syncthreads();   // the warps' s1 rows are complete
    if (tid < D) {
      float t = 0.f;
      for (int w2 = 0; w2 < kGrWarps; ++w2) t += s1_row(w2)[tid];
      P[D * D + tid] = t;
    }
    q += ntile;
    cc += nchunk;
    T = Te;
    fence_before();
    ok = !__syncthreads_or(*abort_flag);   // the sum's reads are done before the next segment; uniform
    fence_after();
  }
  fence_before();
  __syncthreads();
  if (warp == kGrMmaWarp) {
    // every issued MMA has landed before TMEM is released (after an abort the
    // epilogue may not have waited for the last chunks)
    if (mma_issued) {
      mma_commit_w(&bar.done);
      drain_bar(&bar.done, 0, a.status);
    }
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(512));
  }
}

// A group's split axis from its Gram partials: grid (2^lvl, B*H), 256 threads.
// G = the sum of the partials (CTA order); C = G - s1 s1^T / n; the power
// steps start from r - mean = -s1 / n (e_0 if that is zero).
__global__ void __launch_bounds__(256) rb_axis_kernel(const ReblockArgs a, int lvl, int tph, int chunk, int iters) {
  constexpr int D = 128, LD = D + 1;
  extern __shared__ __align__(16) float G[];   // [D][LD]
  __shared__ float s1[D], w[D], z[D];
  __shared__ float s_tmp;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y, grp = blockIdx.x;
  int start, len;
  if (!rb_segment(a.n_v, lvl, grp, start, len) || len <= kBlock) return;
  const int64_t gidx = ((int64_t)bh << lvl) + grp;
  const int c0 = (bh * tph + start / kGrRows) / chunk, c1 = (bh * tph + (start + len - 1) / kGrRows) / chunk;
  {   // thread tid sums float4 f = tid + 256 k (k < 16) of every partial, 16 loads in flight
    float4 acc[D * D / 4 / 256];
#pragma unroll
    for (int k = 0; k < D * D / 4 / 256; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = c0; c <= c1; ++c) {
      const float4* src = reinterpret_cast<const float4*>(a.gpart + (size_t)(gidx + c) * kGramPartFloats);
#pragma unroll
      for (int k = 0; k < D * D / 4 / 256; ++k) {
        const float4 v = src[tid + 256 * k];
        acc[k].x += v.x; acc[k].y += v.y; acc[k].z += v.z; acc[k].w += v.w;
      }
    }
#pragma unroll
    for (int k = 0; k < D * D / 4 / 256; ++k) {
      const int idx = 4 * (tid + 256 * k), i = idx / D, j = idx % D;
      G[i * LD + j] = acc[k].x; G[i * LD + j + 1] = acc[k].y; G[i * LD + j + 2] = acc[k].z; G[i * LD + j + 3] = acc[k].w;
    }
  }
  const float inv_n = 1.f / (float)len;
  if (tid < D) {
    float t = 0.f;
    for (int c = c0; c <= c1; ++c) t += a.gpart[(size_t)(gidx + c) * kGramPartFloats + D * D + tid];
    s1[tid] = t;
    // r - mean = (r - c) - s1 / n; the mean c + s1 / n is the children's shift
    const float cv = a.cbuf[rb_shift_index(a, lvl, bh, grp) * D + tid];
    const float r = a.Y[((int64_t)bh * a.n_v + a.ord[(int64_t)bh * a.n_v + start]) * D + tid];
    w[tid] = (r - cv) - t * inv_n;
    a.cbuf[rb_shift_index(a, lvl + 1, bh, 2 * grp) * D + tid] = cv + t * inv_n;
  }
  __syncthreads();
  {
    const float n0 = rb_norm(w, D, &s_tmp);
    if (tid < D) w[tid] = n0 > 0.f ? w[tid] / n0 : (tid == 0 ? 1.f : 0.f);
    __syncthreads();
  }
  for (int it = 0; it < iters; ++it) {
    if (warp == 0) {   // s1 . w
      float t = 0.f;
      for (int i = lane; i < D; i += 32) t = fmaf(s1[i], w[i], t);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) s_tmp = t * inv_n;
    }
    __syncthreads();
    if (tid < D) {
      float t = 0.f;
      for (int j = 0; j < D; ++j) t = fmaf(G[tid * LD + j], w[j], t);
      z[tid] = t - s1[tid] * s_tmp;
    }
    __syncthreads();
    const float nz = rb_norm(z, D, &s_tmp);
    if (!(nz > 0.f)) break;   // uniform
    if (tid < D) w[tid] = z[tid] / nz;
    __syncthreads();
  }
  if (tid < D) a.wbuf[gidx * D + tid] = w[tid];
}

// One level of the hierarchy: grid (2^lvl NC, B*H); group blockIdx.x / NC of every head.
// With NC > 1 the NC CTAs of a cluster share the group: each streams the contiguous
// slice [lo, hi) of its positions, and the block sums, the radix histograms and the
// partition's left/right counts are summed over the cluster in rank order through
// distributed shared memory, so every CTA holds the same mean, axis and pivot.
// With kAxis the group's split axis is read from a.wbuf (rb_axis_kernel), and
// only the projection pass streams the rows.
template <int D, int T, int NC, bool kAxis>
__device__ __forceinline__ void rb_split_group(const ReblockArgs& a, int lvl, int iters) {
  constexpr int kSplitThreads = T, kSplitWarps = T / 32;
  constexpr int LPR = D / 4, RPW = 32 / LPR, SLOTS = kSplitWarps * RPW;
  __shared__ __align__(16) float4 red[kSplitWarps][LPR];
  __shared__ uint32_t wsum[8];
  __shared__ __align__(16) float mean[D], w[D], z[D];
  __shared__ uint32_t hist[256];
  __shared__ int s_int[4];
  __shared__ float s_tmp;
  __shared__ __align__(16) float part[NC > 1 ? D : 1];      // this CTA's share of a block sum
  __shared__ uint32_t htot[NC > 1 ? 256 : 1];               // the cluster's histogram
  __shared__ int s_cnt[2];                                  // this CTA's left / right counts
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane / LPR, fl = lane % LPR;   // row slot within the warp, lane quad of the row
  const int bh = blockIdx.y;
  const int grp = blockIdx.x / NC, rank = blockIdx.x % NC;
  int start, len;
  if (!rb_segment(a.n_v, lvl, grp, start, len) || len <= kBlock) return;   // uniform over the cluster
  const int left = rb_left(len);
  const int lo = (int)((int64_t)len * rank / NC), hi = (int)((int64_t)len * (rank + 1) / NC);
  // a block sum of a per-lane float4 over the CTA, then over the cluster (rank order)
  auto cluster_sum = [&](float4 v, float* out, float scale) {
    if constexpr (NC == 1) {
      rb_block_sum<D, kSplitWarps>(v, red, out, scale);
    } else {
      namespace cg = cooperative_groups;
      cg::cluster_group cluster = cg::this_cluster();
      rb_block_sum<D, kSplitWarps>(v, red, part, 1.f);
      cluster.sync();
      if (tid < D) {
        float t = 0.f;
        for (int r = 0; r < NC; ++r) t += cluster.map_shared_rank(part, r)[tid];
        out[tid] = t * scale;
      }
      cluster.sync();   // every CTA has read every part; out is visible to the block
    }
  };
  int32_t* ord = a.ord + (int64_t)bh * a.n_v + start;
  const float* Y = a.Y + (int64_t)bh * a.n_v * D;
  unsigned long long* key = reinterpret_cast<unsigned long long*>(a.key) + (int64_t)bh * a.n_v + start;

  // pass over the group's rows, U rows of a slot in flight (8 when the projections are the
  // only pass: fewer live values then); the loop bound is warp-uniform, so the row dot
  // products' shuffles see every lane
  constexpr int U = kAxis ? 2 * kSplitUnroll : kSplitUnroll;
  auto rows_pass = [&](auto&& body) {
    for (int w0 = lo + warp * RPW; w0 < hi; w0 += SLOTS * U) {
      int id[U];
      float4 y[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int m = w0 + sub + u * SLOTS;
        id[u] = m < hi ? ord[m] : -1;
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        y[u] = id[u] >= 0 ? *reinterpret_cast<const float4*>(Y + (int64_t)id[u] * D + 4 * fl)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < U; ++u) body(w0 + sub + u * SLOTS, id[u], y[u]);
    }
  };

  if constexpr (kAxis) {
    if (tid < D) w[tid] = a.wbuf[(((int64_t)bh << lvl) + grp) * D + tid];
    __syncthreads();
  } else {
  // mean
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  rows_pass([&](int, int id, float4 y) {
    if (id >= 0) { acc.x += y.x; acc.y += y.y; acc.z += y.z; acc.w += y.w; }
  });
  cluster_sum(acc, mean, 1.f / (float)len);
  // start: the first row minus the mean, normalised (e_0 if that is zero)
  if (tid < D) w[tid] = Y[(int64_t)ord[0] * D + tid] - mean[tid];
  __syncthreads();
  {
    const float n0 = rb_norm(w, D, &s_tmp);
    if (tid < D) w[tid] = n0 > 0.f ? w[tid] / n0 : (tid == 0 ? 1.f : 0.f);
    __syncthreads();
  }
  // power steps on the covariance: z = sum (y - mean) ((y - mean) . w)
  for (int it = 0; it < iters; ++it) {
    const float4 mq = *reinterpret_cast<const float4*>(&mean[4 * fl]);
    const float4 wq = *reinterpret_cast<const float4*>(&w[4 * fl]);
    float4 zq = make_float4(0.f, 0.f, 0.f, 0.f);
    rows_pass([&](int, int id, float4 y) {
      const float4 c = make_float4(y.x - mq.x, y.y - mq.y, y.z - mq.z, y.w - mq.w);
      const float p = rb_row_dot<D>(c, wq);
      if (id >= 0) { zq.x = fmaf(c.x, p, zq.x); zq.y = fmaf(c.y, p, zq.y); zq.z = fmaf(c.z, p, zq.z); zq.w = fmaf(c.w, p, zq.w); }
    });
    cluster_sum(zq, z, 1.f);
    const float nz = rb_norm(z, D, &s_tmp);
    if (!(nz > 0.f)) break;   // uniform
    if (tid < D) w[tid] = z[tid] / nz;
    __syncthreads();
  }
  }
  // projections as 64-bit keys: order-preserving float bits, then the row
  {
    const float4 wq = *reinterpret_cast<const float4*>(&w[4 * fl]);
    rows_pass([&](int m, int id, float4 y) {
      const float p = rb_row_dot<D>(y, wq) + 0.f;   // + 0: -0 -> +0 (ties then go by row)
      if (id >= 0 && fl == 0) {
        const uint32_t u = __float_as_uint(p);
        const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
        key[m] = ((unsigned long long)o << 32) | (uint32_t)id;
      }
    });
  }
  __syncthreads();
  // radix select of the key of rank left-1 (keys are distinct: the row is in them);
  // once the chosen digit's bin holds one key, that key is the only one with the
  // prefix, so "key <= prefix with every lower bit set" selects the same rows
  unsigned long long prefix = 0ull, pmask = 0ull;
  int want = left - 1;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = tid; i < 256; i += kSplitThreads) hist[i] = 0u;
    __syncthreads();
    // warp-aggregated counts: the lanes holding one digit add it once (the top
    // digits of nearby projections coincide, so plain atomics would serialise)
    for (int m0 = lo + warp * 32; m0 < hi; m0 += kSplitThreads) {
      const int m = m0 + lane;
      uint32_t dig = 256u;
      if (m < hi) {
        const unsigned long long k = key[m];
        if ((k & pmask) == prefix) dig = (uint32_t)((k >> shift) & 255ull);
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, dig);
      if (dig < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[dig], (uint32_t)__popc(peers));
    }
    __syncthreads();
    const uint32_t* hs = hist;
    if constexpr (NC > 1) {   // the cluster's histogram, summed in rank order
      namespace cg = cooperative_groups;
      cg::cluster_group cluster = cg::this_cluster();
      cluster.sync();
      for (int i = tid; i < 256; i += kSplitThreads) {
        uint32_t t = 0u;
        for (int r = 0; r < NC; ++r) t += cluster.map_shared_rank(hist, r)[i];
        htot[i] = t;
      }
      cluster.sync();   // every CTA has read every histogram before the next pass clears its own
      hs = htot;
    }
    // the bin holding rank `want`: a parallel exclusive scan of the 256 counts
    uint32_t c = 0u, incl = 0u;
    if (tid < 256) {   // warps 0-7, whole warps
      c = hs[tid];
      incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) wsum[warp] = incl;
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t base = 0u;
      for (int w2 = 0; w2 < warp; ++w2) base += wsum[w2];
      const uint32_t excl = base + incl - c;
      if (excl <= (uint32_t)want && (uint32_t)want < excl + c) {
        s_int[0] = tid;
        s_int[1] = want - (int)excl;
        s_int[2] = (int)c;
      }
    }
    __syncthreads();
    prefix |= (unsigned long long)s_int[0] << shift;
    pmask |= 255ull << shift;
    want = s_int[1];
    const bool single = s_int[2] == 1;   // uniform (over the cluster too: the histograms are the same)
    __syncthreads();
    if (single) break;
  }
  const unsigned long long pivot = prefix | ~pmask;
  // stable partition into tmp: rows with key <= pivot first, in their order
  int32_t* tmp = a.tmp + (int64_t)bh * a.n_v + start;
  int base_l = 0, base_r = left, total_l = 0;
  if constexpr (NC > 1) {   // this CTA's offsets: the left / right counts of the ranks before it
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    int nl = 0;
    for (int m = lo + tid; m < hi; m += kSplitThreads) nl += key[m] <= pivot ? 1 : 0;
    nl = __reduce_add_sync(0xffffffffu, (unsigned)nl);
    if (tid == 0) s_cnt[0] = 0;
    __syncthreads();
    if (lane == 0) atomicAdd(&s_cnt[0], nl);
    __syncthreads();
    if (tid == 0) s_cnt[1] = (hi - lo) - s_cnt[0];
    cluster.sync();
    for (int r = 0; r < NC; ++r) {
      const int* rc = cluster.map_shared_rank(s_cnt, r);
      if (r < rank) { base_l += rc[0]; base_r += rc[1]; }
      total_l += rc[0];
    }
    cluster.sync();   // every CTA has read every count
  }
  for (int c0 = lo; c0 < hi; c0 += kSplitThreads) {
    const int m = c0 + tid;
    const bool valid = m < hi;
    const bool f = valid && key[m] <= pivot;
    const uint32_t bl = __ballot_sync(0xffffffffu, f), bv = __ballot_sync(0xffffffffu, valid);
    const uint32_t below = (1u << lane) - 1u;
    if (lane == 0) { hist[warp] = __popc(bl); hist[32 + warp] = __popc(bv & ~bl); }
    __syncthreads();
    if (warp == 0) {   // exclusive offsets of the warps' counts: one shuffle scan
      const int l2 = lane < kSplitWarps ? (int)hist[lane] : 0, r2 = lane < kSplitWarps ? (int)hist[32 + lane] : 0;
      int il = l2, ir = r2;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yl = __shfl_up_sync(0xffffffffu, il, o), yr = __shfl_up_sync(0xffffffffu, ir, o);
        if (lane >= o) { il += yl; ir += yr; }
      }
      if (lane < kSplitWarps) { hist[64 + lane] = (uint32_t)(il - l2); hist[96 + lane] = (uint32_t)(ir - r2); }
      if (lane == 31) { s_int[2] = il; s_int[3] = ir; }
    }
    __syncthreads();
    if (valid) {
      const int dst = f ? base_l + (int)hist[64 + warp] + __popc(bl & below)
                        : base_r + (int)hist[96 + warp] + __popc(bv & ~bl & below);
      tmp[dst] = ord[m];
    }
    base_l += s_int[2];
    base_r += s_int[3];
    __syncthreads();
  }
  if constexpr (NC > 1) {
    namespace cg = cooperative_groups;
    cg::this_cluster().sync();   // every CTA's rows are in tmp (release / acquire at cluster scope)
  } else {
    total_l = base_l;
  }
  for (int m = lo + tid; m < hi; m += kSplitThreads) ord[m] = tmp[m];
  if (tid == 0 && total_l != left) raise_status(a.status, SOL_ERR_INVALID_ARG);   // cannot happen: keys are distinct
}

template <int D, int T, bool kAxis>
__global__ void __launch_bounds__(T) rb_split_kernel(const ReblockArgs a, int lvl, int iters) {
  rb_split_group<D, T, 1, kAxis>(a, lvl, iters);
}

// Groups larger than the SM count can cover: NC CTAs of 1,024 threads per group, one cluster each.
template <int D, int NC, bool kAxis>
__global__ void __cluster_dims__(NC, 1, 1) __launch_bounds__(1024) rb_split_cluster_kernel(const ReblockArgs a, int lvl,
                                                                                            int iters) {
  rb_split_group<D, 1024, NC, kAxis>(a, lvl, iters);
}


__global__ void rb_perm_kernel(const ReblockArgs a) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)a.B * a.H * a.N;
  if (i >= total) return;
  const int bh = (int)(i / a.N), pos = (int)(i % a.N);
  a.perm[i] = pos < a.n_fix ? pos : a.n_fix + a.ord[(int64_t)bh * a.n_v + pos - a.n_fix];
}

// xp[b, h, pos] = x[b, perm[b, h, pos], h] (gather) or the reverse (scatter):
// D/8 lanes per row, 16 bytes each, so a warp moves 2 (D = 128) or 4 rows.
template <int D, bool kGather>
__global__ void __launch_bounds__(256) rb_rows_kernel(const int32_t* perm, const __nv_bfloat16* src, __nv_bfloat16* dst,
                                                      int B, int H, int N, int64_t sb, int64_t sn, int64_t sh, int* status) {
  constexpr int LPR = D / 8, RPW = 32 / LPR, RPB = 8 * RPW;   // lanes per row, rows per warp, rows per block
  const int lane = threadIdx.x & 31, fl = lane % LPR;
  const int64_t row = (int64_t)blockIdx.x * RPB + (threadIdx.x >> 5) * RPW + lane / LPR;
  if (row >= (int64_t)B * H * N) return;
  const int bh = (int)(row / N), b = bh / H, h = bh % H;
  const int t = perm[row];
  if (t < 0 || t >= N) { if (fl == 0) raise_status(status, SOL_ERR_INVALID_ARG); return; }
  const int64_t strided = (int64_t)b * sb + (int64_t)t * sn + (int64_t)h * sh + fl * 8;
  const int64_t packed = row * D + fl * 8;
  const __nv_bfloat16* s = src + (kGather ? strided : packed);
  __nv_bfloat16* d = dst + (kGather ? packed : strided);
  *reinterpret_cast<uint4*>(d) = *reinterpret_cast<const uint4*>(s);
}

}  // namespace

int reblock_levels(int n_v) {
  int lv = 0;
  for (int leaves = (n_v + kBlock - 1) / kBlock; leaves > 1; leaves = (leaves + 1) / 2) ++lv;
  return lv;
}

int reblock_moment_chunks(int n_q) { return (n_q + kMomRows - 1) / kMomRows; }

int reblock_gram_levels(int n_v, int D) {
  if (D != 128) return 0;
  const int levels = reblock_levels(n_v);
  int g = 0;
  while (g < levels && (n_v >> g) >= kGramMinRows) ++g;
  return g;
}

size_t reblock_gram_part_floats(int BH, int n_v, int D) {
  const int g = reblock_gram_levels(n_v, D);
  return g == 0 ? 0 : (((size_t)BH << (g - 1)) + kGrCtas) * kGramPartFloats;
}

size_t reblock_axis_floats(int BH, int n_v, int D) {
  const int g = reblock_gram_levels(n_v, D);
  return g == 0 ? 0 : ((size_t)BH << (g - 1)) * 128;
}

cudaError_t launch_reblock(const ReblockArgs& a, int iters, cudaStream_t st) {
  const int BH = a.B * a.H;
  if (BH == 0 || a.N == 0) return cudaSuccess;
  const int D = a.D;
  static std::atomic<int> prepared[64];   // once per device: shared-memory opt-in
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int f128 = 128 * 129 * 4, w128 = (128 * 128 + 64 * 129 + 8 * 64) * 4, f64 = 64 * 65 * 4,
            w64 = (64 * 64 + 64 * 65 + 8 * 64) * 4;
  if (dev < 0 || dev >= 64 || !prepared[dev].load(std::memory_order_acquire)) {
    if ((e = cudaFuncSetAttribute(rb_factor_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, f128)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(rb_whiten_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, w128)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(rb_factor_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, f64)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(rb_whiten_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, w64)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(rb_moment_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMomTcSmem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(rb_whiten_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWhTcSmem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(rb_gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGrSmem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(rb_axis_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 129 * 4)) != cudaSuccess)
      return e;
    if (dev >= 0 && dev < 64) prepared[dev].store(1, std::memory_order_release);
  }
  if (a.n_v > 0) {
    // q and k as 4-D [B, N, H, D] maps (the same strides): TMA boxes of 64 dims
    const cuuint64_t bstride = (cuuint64_t)(a.B > 1 ? a.sb : (int64_t)a.N * a.sn) * 2;
    const cuuint64_t dims4[4] = {(cuuint64_t)D, (cuuint64_t)a.H, (cuuint64_t)a.N, (cuuint64_t)a.B};
    const cuuint64_t str4[3] = {(cuuint64_t)a.sh * 2, (cuuint64_t)a.sn * 2, bstride};
    dim3 gm(a.mchunks, BH), gw((a.n_v + kBlock * kWhTiles - 1) / (kBlock * kWhTiles), BH);
    if (D == 128) {
      // the query map of the partial-moment kernel: 64 dims x 64 rows per box, SW128
      CUtensorMap mq;
      const cuuint32_t box4[4] = {64, 1, kMomTcRows, 1};
      if (!make_map(&mq, a.q, 4, dims4, str4, box4, kSw128)) return cudaErrorInvalidValue;
      rb_moment_tc_kernel<<<gm, 128, kMomTcSmem, st>>>(mq, a);
      rb_factor_kernel<128><<<BH, 256, f128, st>>>(a);
      CUtensorMap mk;   // 128-row key tiles of the whitening: 64 dims x 128 rows per box, SW128
      const cuuint32_t boxk[4] = {64, 1, kWhTcRows, 1};
      if (!make_map(&mk, a.k, 4, dims4, str4, boxk, kSw128)) return cudaErrorInvalidValue;
      const int wtph = (a.n_v + kWhTcRows - 1) / kWhTcRows;
      const int wchunk = (BH * wtph + kWhTcCtas - 1) / kWhTcCtas;
      rb_whiten_tc_kernel<<<(BH * wtph + wchunk - 1) / wchunk, kWhTcThreads, kWhTcSmem, st>>>(mk, a, wtph, wchunk);
    } else {
      rb_moment_kernel<64><<<gm, 256, 0, st>>>(a);
      rb_factor_kernel<64><<<BH, 256, f64, st>>>(a);
      rb_whiten_kernel<64><<<gw, 256, w64, st>>>(a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int levels = reblock_levels(a.n_v);
    const int tph = (a.n_v + kGrRows - 1) / kGrRows;   // 64-row tiles per head
    const int chunk = (BH * tph + kGrCtas - 1) / kGrCtas, ngr = (BH * tph + chunk - 1) / chunk;
    for (int lvl = 0; lvl < levels; ++lvl) {
      dim3 gs(1u << lvl, BH);
      const bool wide = (a.n_v >> lvl) > 4096;   // large groups: 1024 threads; small ones: 256, more CTAs per SM
      // fewer groups than SMs: two CTAs of one cluster per group
      const bool pair = wide && (int64_t)BH << lvl < 148;
      if (lvl < a.gram_levels) {   // D = 128: axes from Gram matrices, then one projection pass
        if (lvl == 0) rb_shift0_kernel<<<BH, 1024, 0, st>>>(a);
        rb_gram_tc_kernel<<<ngr, kGrThreads, kGrSmem, st>>>(a, lvl, tph, chunk);
        rb_axis_kernel<<<gs, 256, 128 * 129 * 4, st>>>(a, lvl, tph, chunk, iters);
        if (pair) rb_split_cluster_kernel<128, 2, true><<<dim3(2u << lvl, BH), 1024, 0, st>>>(a, lvl, iters);
        else if (wide) rb_split_kernel<128, 1024, true><<<gs, 1024, 0, st>>>(a, lvl, iters);
        else rb_split_kernel<128, 256, true><<<gs, 256, 0, st>>>(a, lvl, iters);
      } else if (D == 128) {
        if (pair) rb_split_cluster_kernel<128, 2, false><<<dim3(2u << lvl, BH), 1024, 0, st>>>(a, lvl, iters);
        else if (wide) rb_split_kernel<128, 1024, false><<<gs, 1024, 0, st>>>(a, lvl, iters);
        else rb_split_kernel<128, 256, false><<<gs, 256, 0, st>>>(a, lvl, iters);
      } else {
        if (wide) rb_split_kernel<64, 1024, false><<<gs, 1024, 0, st>>>(a, lvl, iters);
        else rb_split_kernel<64, 256, false><<<gs, 256, 0, st>>>(a, lvl, iters);
      }
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  const int64_t total = (int64_t)BH * a.N;
  rb_perm_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_rows(const int32_t* perm, const __nv_bfloat16* src, __nv_bfloat16* dst, int B, int H, int N, int D,
                        int64_t sb, int64_t sn, int64_t sh, bool gather, int* status, cudaStream_t st) {
  const int64_t rows = (int64_t)B * H * N;
  if (rows == 0) return cudaSuccess;
  const int rpb = 8 * (32 / (D / 8));   // rows per 256-thread block
  const unsigned grid = (unsigned)((rows + rpb - 1) / rpb);
  if (D == 128) {
    if (gather) rb_rows_kernel<128, true><<<grid, 256, 0, st>>>(perm, src, dst, B, H, N, sb, sn, sh, status);
    else rb_rows_kernel<128, false><<<grid, 256, 0, st>>>(perm, src, dst, B, H, N, sb, sn, sh, status);
  } else {
    if (gather) rb_rows_kernel<64, true><<<grid, 256, 0, st>>>(perm, src, dst, B, H, N, sb, sn, sh, status);
    else rb_rows_kernel<64, false><<<grid, 256, 0, st>>>(perm, src, dst, B, H, N, sb, sn, sh, status);
  }
  return cudaGetLastError();
}

}  // namespace sol
