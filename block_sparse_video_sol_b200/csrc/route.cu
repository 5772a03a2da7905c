// sol_route kernels: block scores, per-row threshold, exact-block bitmap,
// then CSR lists (exclusive scan of row counts + compaction).
//
// Routing follows the thakicloud blog "MiniMax-H3 ComfyUI accel stack",
// section 이 기술은 무엇인가 (tau counts standard deviations above the mean of
// the block scores), and the Star7 README "MiniMax H3 Activation Chunk &
// Attention Acceleration", section 工作原理 > Sol (Q64/K64 threshold routing,
// prefix KV sink, dense prefix query rows).
//
// The score S = s * qbar kbar^T is a small contraction (2*nqb*nkb*D flop per
// head) compared against a threshold, so it needs fp32 accuracy: TF32 would
// put ~1e-3 relative error on it.  Threshold routing with D = 128 and at most
// 1024 key blocks (route_tc_kernel) runs it on the tensor cores with each
// operand split into two bf16 terms, the score tile held in TMEM.  The other
// cases (Top-K, D = 64) use route_kernel on the fp32
// FMA pipe: one CTA owns 32 query blocks of one (b, h) and all key blocks and
// keeps its 32 x nkb score rows in shared memory, so that the mean, the
// population std and the mask come from one evaluation of S.
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

// Threshold routing with the scores on the tensor cores (D = 128, n_kb <= 1024):
// grid (ceil(n_qb / 128), B*H), 512 threads; query block i0 + r is TMEM lane r.
// q̄ and k̄ (fp32) are each split into two bf16 terms, h = bf16(x) and
// m = bf16(x - h), and S = s·(qh·kh + qh·km + qm·kh) accumulates in fp32 in TMEM:
// the products of bf16 values are exact, and what is left out (the rest of each
// operand below 2^-17 of it, and qm·km below 2^-18) is under 4·10^-6 of |q̄||k̄|s,
// far inside the 10^-4 band in which the routing decision is allowed to differ
// from the fp64 reading.  The 128 × n_kb score tile fills at most the 512 TMEM
// columns, so the row statistics and the mask are taken from TMEM, four threads
// per row (a quarter of its columns each): the mean, the population std (two
// passes, as in route_kernel), then the mask words of the row, 32 columns at a time.
// Past 512 key blocks TMEM holds one half of the row at a time, and each half's
// scores are computed again where a pass needs them (four MMA passes in all).  k̄ is converted in chunks of 128
// key blocks into two shared-memory buffers, so the next chunk's conversion runs
// beside the current chunk's MMAs.
constexpr int kRtRows = 128;
constexpr int kRtThreads = 512;              // all convert; warps 0-3 (TMEM lanes 0-127) take the rows
constexpr int kRtTerm = kRtRows * 128 * 2;   // 32 KB: one bf16 term of a 128-row tile (two 16 KB chunks of 64 dims)
struct RtBars {
  uint64_t mma[2];
  uint32_t tmem;
  int abort_flag;
};
constexpr size_t kRtSmem = 1024 + 2 * kRtTerm + 2 * 2 * kRtTerm + sizeof(RtBars);

// rows [r0, r0 + 128) of x (fp32 [rows][128], rows >= nrows read as zeros) as two bf16 terms,
// K-major SW128: row r's dims 8u .. 8u+7 in chunk u / 8 at 16-byte position (u % 8) ^ (r & 7).
// Thread t handles the 8-dim units t + kRtThreads k; rt_load issues all of its loads at once
// and rt_store splits and writes them, so other work can sit between the two.
constexpr int kRtPer = kRtRows * 16 / kRtThreads;
struct RtLoad { float4 v[kRtPer][2]; };
__device__ __forceinline__ RtLoad rt_load(const float* x, int r0, int nrows) {
  RtLoad l;
#pragma unroll
  for (int k = 0; k < kRtPer; ++k) {
    const int idx = threadIdx.x + kRtThreads * k, r = idx >> 4, u = idx & 15;
    l.v[k][0] = l.v[k][1] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < nrows) {
      l.v[k][0] = *reinterpret_cast<const float4*>(x + (int64_t)(r0 + r) * 128 + 8 * u);
      l.v[k][1] = *reinterpret_cast<const float4*>(x + (int64_t)(r0 + r) * 128 + 8 * u + 4);
    }
  }
  return l;
}
__device__ __forceinline__ void rt_store(const RtLoad& l, uint8_t* th, uint8_t* tm) {
#pragma unroll
  for (int k = 0; k < kRtPer; ++k) {
    const int idx = threadIdx.x + kRtThreads * k, r = idx >> 4, u = idx & 15;
    const float v[8] = {l.v[k][0].x, l.v[k][0].y, l.v[k][0].z, l.v[k][0].w, l.v[k][1].x, l.v[k][1].y, l.v[k][1].z, l.v[k][1].w};
    uint32_t wh[4], wm[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[e], v[e + 1]);
      const __nv_bfloat162 m = __floats2bfloat162_rn(v[e] - __low2float(h), v[e + 1] - __high2float(h));
      wh[e / 2] = *reinterpret_cast<const uint32_t*>(&h);
      wm[e / 2] = *reinterpret_cast<const uint32_t*>(&m);
    }
    const int off = (u >> 3) * (kRtTerm / 2) + r * 128 + (((u & 7) ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(th + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    *reinterpret_cast<uint4*>(tm + off) = make_uint4(wm[0], wm[1], wm[2], wm[3]);
  }
}

__global__ void __launch_bounds__(kRtThreads, 1) route_tc_kernel(const RouteArgs a) {
  constexpr int D = 128;
  extern __shared__ uint8_t rt_smem_raw[];
  uint8_t* qt = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rt_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kt = qt + 2 * kRtTerm;   // [2 buffers][2 terms]
  RtBars& bar = *reinterpret_cast<RtBars*>(kt + 4 * kRtTerm);
  volatile int* abort_flag = &bar.abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, i0 = blockIdx.x * kRtRows;
  const int nch = (a.nkb + kRtRows - 1) / kRtRows;   // 128-block chunks of k̄ (<= 8)
  const float* qbar = a.qbar + (int64_t)bh * a.nqb * D;
  const float* kbar = a.kbar + (int64_t)bh * a.nkb * D;
  if (tid == 0) {
    mbar_init(&bar.mma[0], 1);
    mbar_init(&bar.mma[1], 1);
    bar.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" :: "r"(smem_u32(&bar.tmem)), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  RtLoad lk0 = rt_load(kbar, 0, a.nkb);   // the first chunk, in flight beside q̄'s tile
  {
    const RtLoad lq = rt_load(qbar, i0, a.nqb);
    rt_store(lq, qt, qt + kRtTerm);
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = bar.tmem;
  constexpr uint32_t id = idesc_bf16(128, 128, 0, 0);   // A = q̄ terms, B = k̄ terms, both K-major
  const uint64_t dqh = sdesc(smem_u32(qt), 16, 1024), dqm = dqh + (uint64_t)(kRtTerm >> 4);
  bool ok = true;
  int gc = 0;   // chunk instances run so far: instance g converts into buffer g & 1, commits to mma[g & 1]
  // The scores of key blocks [512 h, 512 h + 512) into TMEM columns 0 .. 511 (chunk j of the
  // half at columns 128 j); every MMA of the half has completed on return (ok uniform).
  int ncommit = 0;   // chunk instances whose MMAs were committed (uniform)
  auto run_half = [&](int h) {
    if (!ok) return;   // uniform
    const int j0 = 4 * h, j1 = min(nch, 4 * h + 4);
    {   // the half's first chunk (its buffer was last read by instance gc - 2, complete by now)
      if (gc == 0) rt_store(lk0, kt, kt + kRtTerm);
      else {
        const RtLoad lk = rt_load(kbar, j0 * kRtRows, a.nkb);
        rt_store(lk, kt + (gc & 1) * 2 * kRtTerm, kt + (gc & 1) * 2 * kRtTerm + kRtTerm);
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the terms feed the tensor cores
    fence_before();
    __syncthreads();   // also: the previous passes' TMEM reads are done before these MMAs
    fence_after();
    for (int j = j0; j < j1; ++j) {
      const int g = gc + (j - j0);
      if (warp == 0) {
        const uint64_t dkh = sdesc(smem_u32(kt + (g & 1) * 2 * kRtTerm), 16, 1024), dkm = dkh + (uint64_t)(kRtTerm >> 4);
        const uint32_t col = tmem + 128 * (j - j0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t o = (uint64_t)(((kk >> 2) * (kRtTerm / 2) + (kk & 3) * 32) >> 4);
          mma_ss_w(col, dqh + o, dkh + o, id, kk > 0 ? 1u : 0u);
          mma_ss_w(col, dqh + o, dkm + o, id, 1u);
          mma_ss_w(col, dqm + o, dkh + o, id, 1u);
        }
        mma_commit_w(&bar.mma[g & 1]);
      }
      ncommit = g + 1;
      if (j + 1 < j1) {   // chunk j+1 into the other buffer, once instance g-1's MMAs have read it
        const RtLoad lk = rt_load(kbar, (j + 1) * kRtRows, a.nkb);   // in flight during the wait
        if (g >= 1) ok = ok && wait_bar(&bar.mma[(g + 1) & 1], ((g - 1) >> 1) & 1, abort_flag, a.status);
        if (ok) rt_store(lk, kt + ((g + 1) & 1) * 2 * kRtTerm, kt + ((g + 1) & 1) * 2 * kRtTerm + kRtTerm);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        fence_before();
        ok = !__syncthreads_or(!ok);
        fence_after();
        if (!ok) break;
      }
    }
    // every chunk's MMAs have landed (commits complete in order: the last one covers all)
    const int gl = gc + (j1 - j0) - 1;
    ok = ok && wait_bar(&bar.mma[gl & 1], (gl >> 1) & 1, abort_flag, a.status);
    ok = !__syncthreads_or(!ok);   // uniform: the TMEM loads that follow are warp-collective
    fence_after();
    gc += j1 - j0;
  };
  // Row passes over the half in TMEM.  Every warp takes part: warp w reads TMEM lanes
  // 32 (w % 4) .. + 31 (rows), and of each row the 32-column pieces pc with pc % 4 == w / 4.
  // The four partial sums of a row are added in shared memory in a fixed order.  Whole
  // warps read TMEM (the loads are warp-collective); rows past n_qb only skip the writes.
  __shared__ float rsum[4][kRtRows];
  __shared__ int rcnt[4][kRtRows];
  const int quad = warp & 3, part = warp >> 2, rr = 32 * quad + lane, i = i0 + rr;
  const uint32_t lane_addr = tmem + ((uint32_t)(32 * quad) << 16);
  const float inv_n = 1.f / (float)a.nkb;
  const bool dense = i < a.n_dense;
  const int64_t row = (int64_t)bh * a.nqb + i;
  const int nh = (nch + 3) / 4;   // halves of up to 512 key blocks (TMEM holds one)
  auto live = [&]() { return ok && i0 + 32 * quad < a.nqb; };   // uniform per warp
  auto pieces = [&](int h) { return (min(a.nkb - 512 * h, 512) + 31) / 32; };
  auto row_total = [&](float x) {   // the four quarters of each row, in order
    rsum[part][rr] = x;
    __syncthreads();
    const float t = (rsum[0][rr] + rsum[1][rr]) + (rsum[2][rr] + rsum[3][rr]);
    __syncthreads();
    return t;
  };
  auto pass_sum = [&](int h) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (live()) {
      for (int pc = part; pc < pieces(h); pc += 4) {
        float v[32];
        tmem_ld32(lane_addr + 32 * pc, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[e & 3] += (512 * h + 32 * pc + e < a.nkb) ? a.scale * v[e] : 0.f;
      }
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
  };
  auto pass_ss = [&](int h, float mu) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (live()) {
      for (int pc = part; pc < pieces(h); pc += 4) {
        float v[32];
        tmem_ld32(lane_addr + 32 * pc, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float t = a.scale * v[e] - mu;
          acc[e & 3] = (512 * h + 32 * pc + e < a.nkb) ? fmaf(t, t, acc[e & 3]) : acc[e & 3];
        }
      }
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
  };
  auto pass_mask = [&](int h, float thr) {
    int cnt = 0;
    if (live()) {
      for (int pc = part; pc < pieces(h); pc += 4) {
        float v[32];
        tmem_ld32(lane_addr + 32 * pc, v);
        tmem_wait_ld();
        uint32_t bits = 0u;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int j = 512 * h + 32 * pc + e;
          const bool sel = j < a.nkb && (dense || j < a.n_sink || a.scale * v[e] > thr);
          bits |= sel ? (1u << e) : 0u;
        }
        if (i < a.nqb) a.mask[row * a.mask_words + 16 * h + pc] = bits;
        cnt += __popc(bits);
      }
    }
    return cnt;
  };
  float mu, sd;
  int cnt;
  if (nh == 1) {   // up to 512 key blocks: one MMA pass, three row passes
    run_half(0);
    mu = row_total(pass_sum(0)) * inv_n;
    sd = sqrtf(row_total(pass_ss(0, mu)) * inv_n);
    const float thr = (a.tau == -INFINITY) ? -INFINITY : fmaf(a.tau, sd, mu);
    cnt = pass_mask(0, thr);
  } else {         // 513-1024: the halves' scores are taken again where a pass needs them
    run_half(0);
    const float s0 = pass_sum(0);
    run_half(1);
    mu = row_total(s0 + pass_sum(1)) * inv_n;
    const float q1 = pass_ss(1, mu);
    run_half(0);
    sd = sqrtf(row_total(pass_ss(0, mu) + q1) * inv_n);
    const float thr = (a.tau == -INFINITY) ? -INFINITY : fmaf(a.tau, sd, mu);
    cnt = pass_mask(0, thr);
    run_half(1);
    cnt += pass_mask(1, thr);
  }
  rcnt[part][rr] = cnt;
  __syncthreads();
  if (live() && part == 0 && i < a.nqb) a.counts[row] = (rcnt[0][rr] + rcnt[1][rr]) + (rcnt[2][rr] + rcnt[3][rr]);
  fence_before();
  __syncthreads();
  if (warp == 0) {
    // after an abort the last committed MMAs may still run: they land before TMEM is released
    if (!ok && ncommit > 0) drain_bar(&bar.mma[(ncommit - 1) & 1], ((ncommit - 1) >> 1) & 1, a.status);
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(512));
  }
}

// Exclusive scan of the row counts in (b, h, i) order by one CTA: warp w owns
// the rows [w c, (w + 1) c) (c a multiple of 32), read 32 at a time (coalesced);
// pass 1 sums them, the warp totals are scanned, pass 2 scans each 32-row step
// with shuffles and carries the running offset.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* counts, int rows, int32_t* row_ptr) {
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = ((rows + 1023) / 1024) * 32;
  const int lo = min(rows, warp * c), hi = min(rows, lo + c);
  int s = 0;
#pragma unroll 4
  for (int r = lo + lane; r < hi; r += 32) s += counts[r];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) warp_tot[warp] = s;
  __syncwarp();   // re-converge the warp first: bar.sync is an aligned barrier
  __syncthreads();
  if (warp == 0) {
    int t = warp_tot[lane], ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    warp_tot[lane] = ti - t;   // exclusive warp offsets
    if (lane == 31) row_ptr[rows] = ti;
  }
  __syncwarp();
  __syncthreads();
  int carry = warp_tot[warp];
#pragma unroll 4
  for (int r0 = lo; r0 < hi; r0 += 32) {   // warp-uniform bounds
    const int r = r0 + lane;
    const int v = r < hi ? counts[r] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (r < hi) row_ptr[r] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
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
        (e = cudaFuncSetAttribute(route_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, max64)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRtSmem)) != cudaSuccess)
      return e;
    if (dev >= 0 && dev < 64) prepared[dev].store(1, std::memory_order_release);
  }
  if (D == 128 && !a.topk && a.nkb <= 8 * kRtRows)   // threshold routing: scores on the tensor cores
    route_tc_kernel<<<dim3((a.nqb + kRtRows - 1) / kRtRows, a.B * a.H), kRtThreads, kRtSmem, st>>>(a);
  else if (D == 128) route_kernel<128><<<grid, 256, smem, st>>>(a, ldS);
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
