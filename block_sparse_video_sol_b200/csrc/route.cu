// sol_route kernels: block scores, per-row threshold, exact-block bitmap,
// then CSR lists (exclusive scan of row counts + compaction).
//
// Routing follows the thakicloud blog "MiniMax-H3 ComfyUI accel stack",
// section 이 기술은 무엇인가 (tau counts standard deviations above the mean of
// the block scores), and the Star7 README "MiniMax H3 Activation Chunk &
// Attention Acceleration", section 工作原理 > Sol (Q64/K64 threshold routing,
// prefix KV sink, dense prefix query rows).
//
// The score S = s * qbar kbar^T is a small fp32 contraction (2*nqb*nkb*D flop
// per head).  It stays on the fp32 FMA pipe: TF32 tensor cores would put
// ~1e-3 relative error on scores that are compared against a threshold.
// One CTA owns 32 query blocks of one (b, h) and all key blocks; it keeps
// its 32 x nkb score rows in shared memory so that the mean, the population
// std and the mask come from one evaluation of S.
//
// The same kernel does Top-K routing: a warp finds each row's k-th largest
// score exactly by a bitwise binary search over order-preserving integer
// keys (counting rounds over the row held in registers, at most 32: it stops
// once exactly k keys lie at or above the candidate), then marks the
// scores above it and, in index order, as many equal to it as k still
// needs.  In the SLA variant (Star7 README, section 工作原理 > SLA, Q=128 /
// K=64 dynamic Top-K) its query rows are 128-row blocks, whose centroid is
// the row-weighted mean of their two 64-row block means, and both 64-row
// halves get the same list; with the compressed branch (the Spark-H3
// configuration) rows are 64-row blocks and the KV sink is kept.
#include <math.h>

#include <atomic>

#include "common.cuh"
#include "ptx.cuh"

namespace sol {

constexpr int kRouteTQ = 32;    // query blocks per CTA
constexpr int kRouteCH = 256;   // key blocks per column chunk
constexpr int kRouteDS = 32;    // head-dim slice held in shared memory
constexpr int kRouteLdK = kRouteCH + 1;  // padded row: conflict-free transposed stores

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Top-K selection for one query row i of the kernel (a 128-row block when
// a.q128, else a 64-row block; one warp; see the file comment); key blocks
// below a.n_sink are kept as well.  Column j = lane + 32 e lives in key[e] (E slots per lane, E*32 >=
// nkb); columns past nkb get key 0, below every real score (order-preserving
// keys of floats are >= 1).
template <int E>
__device__ __forceinline__ void topk_row(const RouteArgs& a, const float* Sr, int i, int bh, int lane) {
  const int nkb = a.nkb, k = a.topk;
  const bool dense = i < a.n_dense;
  uint32_t key[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int j = lane + 32 * e;
    const uint32_t u = j < nkb ? __float_as_uint(Sr[j]) : 0u;
    key[e] = j < nkb ? ((u & 0x80000000u) ? ~u : (u | 0x80000000u)) : 0u;
  }
  uint32_t p = 0u;   // the k-th largest key: the largest v with #{key >= v} >= k
  int need = 0;      // how many keys equal to p are still to be taken
  bool all_eq = false;   // every key equal to p is taken
  if (!dense) {      // uniform over the warp
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = p | (1u << bit);
      int c = 0;
#pragma unroll
      for (int e = 0; e < E; ++e) c += key[e] >= cand ? 1 : 0;
      const int tot = (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
      if (tot >= k) {
        p = cand;
        // exactly k keys >= cand: they are the k largest and the next one is
        // smaller, so {key >= cand} is the selection and no tie is left to break
        if (tot == k) { all_eq = true; break; }
      }
    }
    if (!all_eq) {
      int gt = 0;
#pragma unroll
      for (int e = 0; e < E; ++e) gt += key[e] > p ? 1 : 0;
      need = k - (int)__reduce_add_sync(0xffffffffu, (unsigned)gt);
    }
  }
  const int64_t row0 = (int64_t)bh * a.nqb + (a.q128 ? 2 * i : i);
  const bool second = a.q128 && 2 * i + 1 < a.nqb;
  int cnt = 0;
#pragma unroll
  for (int w = 0; w < E; ++w) {
    if (w < a.mask_words) {   // uniform
      const bool valid = lane + 32 * w < nkb;
      const bool eq = valid && key[w] == p;
      const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
      const int before = __popc(eqb & ((1u << lane) - 1u));
      const bool sel = valid && (dense || lane + 32 * w < a.n_sink || key[w] > p || (eq && (all_eq || before < need)));
      need -= __popc(eqb);
      const uint32_t bits = __ballot_sync(0xffffffffu, sel);
      if (lane == 0) {
        a.mask[row0 * a.mask_words + w] = bits;
        if (second) a.mask[(row0 + 1) * a.mask_words + w] = bits;
      }
      cnt += __popc(bits);
    }
  }
  if (lane == 0) {
    a.counts[row0] = cnt;
    if (second) a.counts[row0 + 1] = cnt;
  }
}

template <int D>
__global__ void __launch_bounds__(256) route_kernel(const RouteArgs a, int ldS) {
  extern __shared__ __align__(16) float sm[];
  float* qT = sm;                          // [D][TQ]
  float* kT = qT + D * kRouteTQ;           // [DS][CH+1]
  float* S = kT + kRouteDS * kRouteLdK;    // [TQ][ldS]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, i0 = blockIdx.x * kRouteTQ;
  const float* qbar = a.qbar + (int64_t)bh * a.nqb * D;
  const float* kbar = a.kbar + (int64_t)bh * a.nkb * D;
  const int nrows = a.q128 ? (a.nqb + 1) / 2 : a.nqb;   // the kernel's query rows

  // Stage q transposed: lane = query row, one float4 of head dims per load;
  // every thread issues all its loads before its first store.
  constexpr int kQv = kRouteTQ * D / 4 / 256;
  {
    float4 qv[kQv];
#pragma unroll
    for (int u = 0; u < kQv; ++u) {
      const int idx = tid + 256 * u, r = idx % kRouteTQ, d = 4 * (idx / kRouteTQ), i = i0 + r;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < nrows) {
        if (a.q128) {   // 128-row block: row-weighted mean of its 64-row block means
          const float n0 = (float)(min(a.N, 128 * i + 64) - 128 * i);
          const float n1 = 2 * i + 1 < a.nqb ? (float)(min(a.N, 128 * i + 128) - (128 * i + 64)) : 0.f;
          const float4 q0 = *reinterpret_cast<const float4*>(qbar + (int64_t)(2 * i) * D + d);
          float4 q1 = make_float4(0.f, 0.f, 0.f, 0.f);
          if (n1 > 0.f) q1 = *reinterpret_cast<const float4*>(qbar + (int64_t)(2 * i + 1) * D + d);
          const float n = n0 + n1;
          v = make_float4((n0 * q0.x + n1 * q1.x) / n, (n0 * q0.y + n1 * q1.y) / n,
                          (n0 * q0.z + n1 * q1.z) / n, (n0 * q0.w + n1 * q1.w) / n);
        } else {
          v = *reinterpret_cast<const float4*>(qbar + (int64_t)i * D + d);
        }
      }
      qv[u] = v;
    }
#pragma unroll
    for (int u = 0; u < kQv; ++u) {
      const int idx = tid + 256 * u, r = idx % kRouteTQ, d = 4 * (idx / kRouteTQ);
      qT[(d + 0) * kRouteTQ + r] = qv[u].x;
      qT[(d + 1) * kRouteTQ + r] = qv[u].y;
      qT[(d + 2) * kRouteTQ + r] = qv[u].z;
      qT[(d + 3) * kRouteTQ + r] = qv[u].w;
    }
  }
  const int rg = warp & 3;   // rows 8*rg .. 8*rg+7
  const int chh = warp >> 2; // columns 128*chh .. +127 of the chunk

  // k slices (kRouteCH key blocks x kRouteDS head dims) are software-pipelined
  // through registers: the next slice's loads are issued before the current
  // slice's FMAs, so their latency hides behind the arithmetic.
  constexpr int kKv = kRouteCH * kRouteDS / 4 / 256;
  float4 kn[kKv];
  auto load_slice = [&](int c0, int d0) {
#pragma unroll
    for (int u = 0; u < kKv; ++u) {
      const int idx = tid + 256 * u, jj = idx / (kRouteDS / 4), dq = (idx % (kRouteDS / 4)) * 4;
      kn[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + jj < a.nkb) kn[u] = *reinterpret_cast<const float4*>(kbar + (int64_t)(c0 + jj) * D + d0 + dq);
    }
  };
  load_slice(0, 0);
  for (int c0 = 0; c0 < a.nkb; c0 += kRouteCH) {
    // acc[p][c]: rows 8*rg + 2p (low half) and 2p+1 (high half) of column c,
    // updated by one packed f32x2 FMA (each half an ordinary fp32 FMA)
    uint64_t acc[4][4];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[p][c] = 0ull;
    for (int d0 = 0; d0 < D; d0 += kRouteDS) {
      __syncwarp();   // re-converge the warp first: bar.sync is an aligned barrier
      __syncthreads();
#pragma unroll
      for (int u = 0; u < kKv; ++u) {
        const int idx = tid + 256 * u, jj = idx / (kRouteDS / 4), dq = (idx % (kRouteDS / 4)) * 4;
        kT[(dq + 0) * kRouteLdK + jj] = kn[u].x;
        kT[(dq + 1) * kRouteLdK + jj] = kn[u].y;
        kT[(dq + 2) * kRouteLdK + jj] = kn[u].z;
        kT[(dq + 3) * kRouteLdK + jj] = kn[u].w;
      }
      __syncwarp();   // re-converge the warp first: bar.sync is an aligned barrier
      __syncthreads();
      {   // the next slice: next head-dim slice, else the next chunk's first
        const int nd0 = d0 + kRouteDS < D ? d0 + kRouteDS : 0;
        const int nc0 = d0 + kRouteDS < D ? c0 : c0 + kRouteCH;
        if (nc0 < a.nkb) load_slice(nc0, nd0);
      }
#pragma unroll
      for (int dd = 0; dd < kRouteDS; ++dd) {
        const float4 qa = *reinterpret_cast<const float4*>(qT + (d0 + dd) * kRouteTQ + 8 * rg);
        const float4 qb = *reinterpret_cast<const float4*>(qT + (d0 + dd) * kRouteTQ + 8 * rg + 4);
        const uint64_t q2[4] = {f2pack(qa.x, qa.y), f2pack(qa.z, qa.w), f2pack(qb.x, qb.y), f2pack(qb.z, qb.w)};
        uint64_t k2[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float kv = kT[dd * kRouteLdK + 128 * chh + lane + 32 * c];
          k2[c] = f2pack(kv, kv);
        }
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[p][c] = ffma2(q2[p], k2[c], acc[p][c]);
      }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col = c0 + 128 * chh + lane + 32 * c;
        float lo, hi;
        f2unpack(acc[p][c], lo, hi);
        if (col < a.nkb) {
          S[(8 * rg + 2 * p) * ldS + col] = a.scale * lo;
          S[(8 * rg + 2 * p + 1) * ldS + col] = a.scale * hi;
        }
      }
  }
  __syncwarp();   // re-converge the warp first: bar.sync is an aligned barrier
  __syncthreads();

  // Row statistics and mask: warp w handles rows 4w .. 4w+3.
  const float inv_n = 1.f / (float)a.nkb;
  for (int rr = 0; rr < kRouteTQ / 8; ++rr) {
    const int r = warp * (kRouteTQ / 8) + rr, i = i0 + r;
    if (i >= nrows) break;
    const float* Sr = S + r * ldS;
    if (a.topk) {   // the row's scores in as few register slots per lane as cover nkb
      if (a.nkb <= 128) topk_row<4>(a, Sr, i, bh, lane);
      else if (a.nkb <= 256) topk_row<8>(a, Sr, i, bh, lane);
      else if (a.nkb <= 512) topk_row<16>(a, Sr, i, bh, lane);
      else topk_row<32>(a, Sr, i, bh, lane);
      continue;
    }
    float s = 0.f;
    for (int j = lane; j < a.nkb; j += 32) s += Sr[j];
    const float mu = warp_sum(s) * inv_n;
    float ss = 0.f;
    for (int j = lane; j < a.nkb; j += 32) { const float t = Sr[j] - mu; ss = fmaf(t, t, ss); }
    const float sd = sqrtf(warp_sum(ss) * inv_n);
    const float thr = (a.tau == -INFINITY) ? -INFINITY : fmaf(a.tau, sd, mu);
    const bool dense = i < a.n_dense;
    const int64_t row = (int64_t)bh * a.nqb + i;
    int cnt = 0;
    for (int w = 0; w < a.mask_words; ++w) {
      const int j = w * 32 + lane;
      const bool sel = j < a.nkb && (dense || j < a.n_sink || Sr[j] > thr);
      const uint32_t bits = __ballot_sync(0xffffffffu, sel);
      if (lane == 0) a.mask[row * a.mask_words + w] = bits;
      cnt += __popc(bits);
    }
    if (lane == 0) a.counts[row] = cnt;
  }
}

// Exclusive scan of the row counts in (b, h, i) order by one CTA.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* counts, int rows, int32_t* row_ptr) {
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (rows + 1023) / 1024;
  const int lo = min(rows, tid * per), hi = min(rows, lo + per);
  int s = 0;
  for (int r = lo; r < hi; ++r) s += counts[r];
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncwarp();   // re-converge the warp first: bar.sync is an aligned barrier
  __syncthreads();
  if (warp == 0) {
    int t = warp_tot[lane], ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    warp_tot[lane] = ti - t;  // exclusive warp offsets
  }
  __syncwarp();   // re-converge the warp first: bar.sync is an aligned barrier
  __syncthreads();
  int run = warp_tot[warp] + incl - s;
  for (int r = lo; r < hi; ++r) { row_ptr[r] = run; run += counts[r]; }
  if (tid == 1023) row_ptr[rows] = warp_tot[31] + incl;
}

// One warp per row: bitmap words -> ascending column indices at row_ptr[row].
__global__ void __launch_bounds__(256) compact_kernel(const uint32_t* mask, const int32_t* row_ptr, int rows,
                                                      int mask_words, int32_t* col_idx) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  int base = row_ptr[row];
  const uint32_t* m = mask + (int64_t)row * mask_words;
  for (int w = 0; w < mask_words; ++w) {
    const uint32_t bits = m[w];
    if ((bits >> lane) & 1u) col_idx[base + __popc(bits & ((1u << lane) - 1u))] = w * 32 + lane;
    base += __popc(bits);
  }
}

static size_t route_smem_bytes(int D, int ldS) {
  return sizeof(float) * ((size_t)D * kRouteTQ + (size_t)kRouteDS * kRouteLdK + (size_t)kRouteTQ * ldS);
}

cudaError_t launch_route(const RouteArgs& a, int D, cudaStream_t st) {
  const int ldS = ((a.nkb + 3) / 4) * 4;
  const size_t smem = route_smem_bytes(D, ldS);
  const int nrows = a.q128 ? (a.nqb + 1) / 2 : a.nqb;
  dim3 grid((nrows + kRouteTQ - 1) / kRouteTQ, a.B * a.H);
  // Shared-memory opt-in once per device, for the largest problem (so that
  // launches stay free of attribute calls, e.g. inside a stream capture).
  static std::atomic<int> prepared[64];   // zero-initialised; set once per device (any thread)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !prepared[dev].load(std::memory_order_acquire)) {
    const int max128 = (int)route_smem_bytes(128, kMaxKeyBlocks), max64 = (int)route_smem_bytes(64, kMaxKeyBlocks);
    if ((e = cudaFuncSetAttribute(route_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, max128)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(route_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, max64)) != cudaSuccess)
      return e;
    if (dev >= 0 && dev < 64) prepared[dev].store(1, std::memory_order_release);
  }
  if (D == 128) route_kernel<128><<<grid, 256, smem, st>>>(a, ldS);
  else route_kernel<64><<<grid, 256, smem, st>>>(a, ldS);
  return cudaGetLastError();
}

cudaError_t launch_scan_compact(const uint32_t* mask, const int32_t* counts, int rows, int mask_words,
                                int32_t* row_ptr, int32_t* col_idx, cudaStream_t st) {
  scan_kernel<<<1, 1024, 0, st>>>(counts, rows, row_ptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  compact_kernel<<<(rows + 7) / 8, 256, 0, st>>>(mask, row_ptr, rows, mask_words, col_idx);
  return cudaGetLastError();
}

}  // namespace sol
