// sol_attn_fwd on sm_100a: exact + centroid attention with TMA, tcgen05 MMAs
// and TMEM accumulators.
//
// Star7 README "MiniMax H3 Activation Chunk & Attention Acceleration",
// section 工作原理 > Sol: the selected K/V blocks of a query block are
// attended exactly; every unselected block contributes one term through its
// K/V centroid (logit s*q.kbar_j + log n_j, value vbar_j; plus the log-mass
// bias of the Spark-H3 news page, Spark-Reweight bullet, when enabled), and
// both kinds of term are merged in the same FP32 online softmax.
//
// Tiling.  A CTA owns one 128-row query tile = two consecutive 64-row query
// blocks (rows 0-63: block i0, rows 64-127: block i0+1) of one (b, h); the
// tcgen05 MMA runs at full rate only with M = 128.  The two blocks route to
// different key blocks, so the CTA walks the sorted union of their CSR lists,
// two key blocks (128 keys) per S tile; each union entry carries a 2-bit tag
// saying which half needs it, and a half that does not need a block gets
// p = 0 there (its exponentials are skipped, warp-uniformly).  Then come the
// centroid tiles: 128 centroids each, the half's selected blocks masked.
//
// Roles (16 warps):
//   warp 0     TMA producer: Q once, then the K tiles into a 3-stage ring.
//   warp 1     MMA issuer (the whole warp; one elected lane issues):
//              S_(t%3) = Q K^T into TMEM, then O += P V with P read from
//              TMEM; QK runs three tiles ahead.
//   warp 2     TMA producer: the V tiles into a 2-stage ring.
//   warps 4-15 softmax warpgroups 0, 1, 2: group g takes the S tiles
//              t = g, g+3, ... (S buffer g).  One thread per row (TMEM
//              lane), fp32 online softmax with lazy rescaling: the groups
//              share each row's reference max (handed from step t-1 to
//              step t through an mbarrier per warp) and O is rescaled only
//              when that reference grows by more than 2^8; bf16 P is
//              written back over S.  The groups rotate, so one group's
//              exponentials overlap the others' TMEM traffic and waits.
//              The epilogue normalises O and stores bf16 rows.
// TMEM: S_0, S_1, S_2 = columns [0,128), [128,256), [256,384) (P = bf16 pairs
//       over the first 64 columns of its S), O = [384, 384+D).
// Every mbarrier wait is bounded; on expiry the kernel raises
// SOL_ERR_TIMEOUT, stops issuing, drains what it issued and frees TMEM.
#include <cuda.h>
#include <math.h>

#include <atomic>

#include "common.cuh"
#include "ptx.cuh"

namespace sol {
namespace {

#ifdef SOL_FAULT_TEST
__device__ int g_drop_p_arrive = -1;   // step whose "P ready" arrive is withheld (-1: none)
#endif

constexpr int kSoftmaxGroups = 3;   // softmax warpgroups: one per S buffer
constexpr int kThreads = 128 * (kSoftmaxGroups + 1);   // + one control warpgroup: 16 warps
constexpr int kKWarp = 0, kMmaWarp = 1, kVWarp = 2;   // warp 3 idles; warps 4-11 softmax
constexpr uint32_t kOCol = 384;     // TMEM column of O; S_0, S_1, S_2 at 0, 128, 256
// Register split (setmaxnreg): the block launches with kRegsLaunch per
// thread; the control warpgroup gives registers back to the softmax
// warpgroups.  kSoftmaxGroups*128*kRegsSoftmax + 128*kRegsControl must not
// exceed kThreads*kRegsLaunch.
constexpr int kRegsLaunch = 128, kRegsSoftmax = 152, kRegsControl = 56;
static_assert(kSoftmaxGroups * 128 * kRegsSoftmax + 128 * kRegsControl <= kThreads * kRegsLaunch, "register split");
constexpr int kKStages = 3;   // K tiles in flight (needed first, by QK)
constexpr int kVStages = 2;   // V tiles in flight (needed a softmax later, by PV)
// A K stage is released by the commit that signals its S buffer and a V stage
// by the commit that signals its PV, so the rings match those buffers.
static_assert(kKStages == 3 && kVStages == 2, "K ring = S buffers, V ring = o_done barriers");

// Optional phase trace (build with -DSOL_TRACE): 32-bit clock() stamps of one
// CTA's roles for its first kTraceSteps S tiles, kept in shared memory (a
// global store before a release-semantics mbarrier arrive would stall it) and
// copied out at the end; read back with sol_debug_trace().
#ifdef SOL_TRACE
constexpr int kTraceSteps = 128;
constexpr int kTraceSlots = 24;
__device__ unsigned int g_trace[kTraceSlots * kTraceSteps];
#ifndef SOL_TRACE_BX
#define SOL_TRACE_BX 0
#endif
#ifndef SOL_TRACE_BY
#define SOL_TRACE_BY 0
#endif
#define SOL_TRACE_ON (blockIdx.x == SOL_TRACE_BX && blockIdx.y == SOL_TRACE_BY && blockIdx.z == 0)
__device__ __forceinline__ unsigned int sol_gtime() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return (unsigned int)t;
}
// globaltimer (ns) stamps of CTA-level events in slot 9, steps 8.. (comparable across warps)
#define SOL_GT_AT(k) do { if (SOL_TRACE_ON) x.trace[9 * kTraceSteps + 8 + (k)] = sol_gtime(); } while (0)
#define SOL_TRACE_AT(slot, step) \
  do { if (SOL_TRACE_ON && (step) < kTraceSteps) x.trace[(slot) * kTraceSteps + (step)] = (unsigned int)clock(); } while (0)
#else
#define SOL_TRACE_AT(slot, step) do { } while (0)
#endif
constexpr float kRescale = 8.0f;   // log2 units: rescale O when the max grows by more than 2^8
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxWords = kMaxKeyBlocks / 32;
constexpr int kMaxCentTiles = kMaxKeyBlocks / 128;

template <int D, bool I8 = false>
struct Cfg {
  static constexpr int kChunks = D / 64;               // 128-byte column chunks per row
  static constexpr int kChunkBytes = 128 * 128;        // one chunk of a 128-row tile
  static constexpr int kTileBytes = 128 * D * 2;       // Q, K or V tile of 128 rows
  // INT8 QK: the query codes (128 rows x D bytes, one 128-byte chunk at D = 128); an exact
  // K stage holds the residual codes of the tile's two key blocks and, after them, the
  // two blocks' bf16 means (the mean term's keys)
  static constexpr int kQ8Bytes = I8 ? 128 * D : 0;
  static constexpr int kK8Bytes = 128 * D;
  static constexpr int kKMeanOff = kK8Bytes;
  static constexpr int kSmemTiles = kTileBytes * (1 + kKStages + kVStages) + kQ8Bytes;
  static_assert(!I8 || (D == 128 && kKMeanOff + 2 * D * 2 <= kTileBytes), "INT8 stage layout");
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKStages], v_full[kVStages];
  uint64_t s_full[3], p_full[3], o_done[2], final_mma;
  uint64_t ref_full[kSoftmaxGroups][4];   // [group][warp]: the group's step published its reference max
  uint64_t q8_ready;                      // INT8 QK: the query codes are in shared memory (softmax threads)
  uint64_t kb_done[kKStages];             // INT8 QK: the softmax has read the stage's block means (4 warps)
};

template <bool I8>
struct Extra {
  Bars bar;
  uint32_t tmem_base;
  int abort_flag;
  int n_union, n_cent, present[2];
  uint32_t sel[2][kMaxWords];        // exact-block bitmaps of the two halves
  int cent[kMaxCentTiles];           // centroid tiles to visit
  int list[kMaxKeyBlocks];           // union entries: j | needA << 16 | needB << 17
  int cent_live[kMaxCentTiles][2][2];           // [slot][half][64-column half]: any live centroid
  // log2-unit offset of each centroid column, -inf if masked (the INT8 variant, short of
  // shared memory, computes it from cbias and the bitmaps instead)
  alignas(16) float cent_add[I8 ? 1 : kMaxCentTiles][2][128];
  float qsig[I8 ? 128 : 1];                     // INT8 QK: each row's query scale
  alignas(16) float tail_add[64];                         // 0 for valid rows of the last key block, -inf beyond N
  float2 ml[kSoftmaxGroups][128];               // per warpgroup and row: (reference, partial sum)
  float m_ref[128];                             // per row: reference max after the latest step (log2 units)
  alignas(16) float cbias[kMaxKeyBlocks];       // this (b, h)'s centroid logit biases, prefetched
#ifdef SOL_TRACE
  unsigned int trace[kTraceSlots * kTraceSteps];
#endif
};

// tcgen05 descriptors, MMA issue, commits and TMEM loads/stores: ptx.cuh.

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Exact float of an s32 stored in a float register (|S| < 2^22): 1.5 * 2^23 + S is a
// float of the same bits plus 0x4B400000, from which 1.5 * 2^23 subtracts exactly.
__device__ __forceinline__ float i2f_exact(float bits) {
  return __int_as_float(__float_as_int(bits) + 0x4B400000) - 12582912.f;
}
__device__ __forceinline__ void bf16x8_f32(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// O row *= f for this warp's 32 rows (rarely executed; kept out of the
// softmax loop's instruction stream).
template <int D>
__device__ __noinline__ void rescale_rows(uint32_t o_addr, float f) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    float ov[32];
    tmem_ld32(o_addr + 32 * c, ov);
    tmem_wait_ld();
    uint32_t ou[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) ou[e] = __float_as_uint(ov[e] * f);
    tmem_st32(o_addr + 32 * c, ou);
  }
}

struct TcParams {
  AttnArgs a;
  int mask_words;
};

// bar.sync is an aligned barrier: every warp must reach it converged, so the
// lanes of warps that ran lane-0-only work (TMA producers, set-up) are
// re-converged first.  Without it a warp whose lanes arrive apart can let the
// barrier complete early.
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  __syncwarp();
  asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void cta_sync() {
  __syncwarp();
  __syncthreads();
}

// ---- plan kernel -------------------------------------------------------------------------------
// Per query tile (two consecutive 64-row query blocks of one (b, h)): the
// exact-block bitmaps of both blocks from their CSR lists, the union of the
// lists with per-half tags, and the centroid tiles to visit, written to the
// tile's plan (layout: plan_ints in common.cuh).  Building this inside the
// attention kernel cost each CTA several microseconds at its start, with the
// tensor cores idle (the set-up code runs once per CTA from a cold
// instruction cache while HBM is saturated); here one warp per tile builds
// it for all tiles at once.  Out-of-range CSR entries raise
// SOL_ERR_INVALID_ARG and are skipped.
constexpr int kPlanWarps = 8;

__global__ void __launch_bounds__(kPlanWarps * 32) plan_kernel(const AttnArgs a, int mw) {
  __shared__ uint32_t sel[kPlanWarps][2][kMaxWords];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntq = (a.nqb + 1) / 2;
  const int64_t tile = (int64_t)blockIdx.x * kPlanWarps + warp;
  if (tile >= (int64_t)a.B * a.H * ntq) return;   // whole warp
  const int tq = (int)(tile % ntq);
  const int64_t bh = tile / ntq;
  const int i0 = 2 * tq;
  for (int w = lane; w < 2 * kMaxWords; w += 32) (&sel[warp][0][0])[w] = 0u;
  __syncwarp();
  for (int hf = 0; hf < 2; ++hf) {
    const int i = i0 + hf;
    if (i >= a.nqb) continue;
    const int64_t row = bh * a.nqb + i;
    const int beg = a.row_ptr[row], end = a.row_ptr[row + 1];
    for (int e = beg + lane; e < end; e += 32) {
      const int j = a.col_idx[e];
      if (j >= 0 && j < a.nkb) atomicOr(&sel[warp][hf][j >> 5], 1u << (j & 31));
      else raise_status(a.status, SOL_ERR_INVALID_ARG);
    }
  }
  __syncwarp();
  int* P = a.plan + tile * plan_ints(mw, a.nkb);
  int* list = P + 16 + 2 * mw;
  // Union list with per-half tags.  The S tiles take consecutive pairs of
  // entries, and a half's exponentials are skipped for a block it does not
  // need, so the order balances the two halves' warps: first pairs (block
  // only A needs, block only B needs), then the blocks both need, then the
  // leftover single-half blocks.  (The online softmax is order-free.)
  const uint32_t ua = lane < mw ? sel[warp][0][lane] : 0u, ub = lane < mw ? sel[warp][1][lane] : 0u;
  const uint32_t oa = ua & ~ub, ob = ub & ~ua, oc = ua & ub;
  const int ca = __popc(oa), cb = __popc(ob), cc = __popc(oc);
  int ia = ca, ib = cb, ic = cc;   // inclusive scans over the lanes' words
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, ia, o), yb = __shfl_up_sync(0xffffffffu, ib, o),
              yc = __shfl_up_sync(0xffffffffu, ic, o);
    if (lane >= o) { ia += ya; ib += yb; ic += yc; }
  }
  const int NA = __shfl_sync(0xffffffffu, ia, 31), NB = __shfl_sync(0xffffffffu, ib, 31),
            NC = __shfl_sync(0xffffffffu, ic, 31);
  const int npair = min(NA, NB), rest = 2 * npair + NC;   // leftovers of one kind start at rest
  int ra = ia - ca, rb = ib - cb, rc = ic - cc;
  for (uint32_t m = oa; m; m &= m - 1, ++ra)
    list[ra < npair ? 2 * ra : rest + ra - npair] = (32 * lane + __ffs(m) - 1) | (1 << 16);
  for (uint32_t m = ob; m; m &= m - 1, ++rb)
    list[rb < npair ? 2 * rb + 1 : rest + rb - npair] = (32 * lane + __ffs(m) - 1) | (1 << 17);
  for (uint32_t m = oc; m; m &= m - 1, ++rc)
    list[2 * npair + rc] = (32 * lane + __ffs(m) - 1) | (3 << 16);
  // centroid tiles (128 blocks = 4 bitmap words) holding at least one
  // block unselected by a present half: lane w checks word w
  const bool present1 = i0 + 1 < a.nqb;
  const uint32_t vm = lane < mw ? (a.nkb - 32 * lane >= 32 ? 0xffffffffu : ((1u << (a.nkb - 32 * lane)) - 1u)) : 0u;
  const uint32_t wb = __ballot_sync(0xffffffffu, ((~ua & vm) != 0u) || (present1 && (~ub & vm) != 0u));
  if (lane < mw) {
    P[16 + lane] = (int)ua;
    P[16 + mw + lane] = (int)ub;
  }
  if (lane == 0) {
    int n = 0;
    for (int ct = 0; ct < 8; ++ct)
      if ((wb >> (4 * ct)) & 0xFu) P[4 + n++] = ct;
    P[0] = NA + NB + NC;
    P[1] = a.centroids ? n : 0;   // Top-K routing without the compressed branch drops unselected blocks
    P[2] = present1 ? 1 : 0;
  }
}

template <int D, bool I8>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
               const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mkb,
               const __grid_constant__ CUtensorMap mvb, const __grid_constant__ CUtensorMap mk8,
               const TcParams prm) {
  using C = Cfg<D, I8>;
  const AttnArgs& a = prm.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::kTileBytes;
  uint8_t* sV = sK + kKStages * C::kTileBytes;
  uint8_t* sQ8 = sV + kVStages * C::kTileBytes;   // INT8 QK: query codes (SW128, 128-byte rows)
  Extra<I8>& x = *reinterpret_cast<Extra<I8>*>(sQ8 + C::kQ8Bytes);
  Bars& bar = x.bar;
  volatile int* abort_flag = &x.abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
#ifdef SOL_TRACE
  const unsigned int t_entry = (unsigned int)clock(), g_entry = sol_gtime();
#endif
  const int tq = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = (int64_t)b * a.H + h;
  const int i0 = 2 * tq;
  const int mw = prm.mask_words;

  // ---- set-up: barriers, TMEM, routing lists --------------------------------------------------
  if (tid == 0) {
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < kKStages; ++s) mbar_init(&bar.k_full[s], 1);
    for (int s = 0; s < kVStages; ++s) mbar_init(&bar.v_full[s], 1);
    for (int s = 0; s < 3; ++s) { mbar_init(&bar.s_full[s], 1); mbar_init(&bar.p_full[s], 4); }
    for (int s = 0; s < 2; ++s) mbar_init(&bar.o_done[s], 1);
    for (int g = 0; g < kSoftmaxGroups; ++g)
      for (int s = 0; s < 4; ++s) mbar_init(&bar.ref_full[g][s], 32);
    mbar_init(&bar.final_mma, 1);
    if (I8) {
      mbar_init(&bar.q8_ready, 128 * kSoftmaxGroups);
      for (int s = 0; s < kKStages; ++s) mbar_init(&bar.kb_done[s], 4);
    }
    x.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // Q does not depend on the routing: its load starts at once
    mbar_expect_tx(&bar.q_full, C::kTileBytes);
    for (int hf = 0; hf < 2; ++hf)
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(sQ + c * C::kChunkBytes + hf * (C::kChunkBytes / 2), &mq, c * 64, h, 64 * (i0 + hf), b, &bar.q_full);
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" :: "r"(smem_u32(&x.tmem_base)), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  const int n_tail = a.N - 64 * (a.nkb - 1);   // valid rows of the last key block
  for (int c = tid; c < 64; c += kThreads) x.tail_add[c] = c < n_tail ? 0.f : -INFINITY;
  // this (b, h)'s centroid biases, needed once the lists are built: loaded now to overlap the CSR reads
  for (int j = tid; j < a.nkb; j += kThreads) x.cbias[j] = a.cbias[bh * a.nkb + j];
#ifdef SOL_TRACE
  for (int i = tid; i < kTraceSlots * kTraceSteps; i += kThreads) x.trace[i] = 0u;
#endif
  cta_sync();
#ifdef SOL_TRACE
  if (tid == 0) SOL_GT_AT(8);
#endif
  {   // this tile's plan (plan_kernel): header, both halves' bitmaps, the union list
    const int* P = a.plan + ((int64_t)bh * ((a.nqb + 1) / 2) + tq) * plan_ints(mw, a.nkb);
    const int n_plan = 16 + 2 * mw + a.nkb;
    for (int e = tid; e < n_plan; e += kThreads) {
      const int v = P[e];
      if (e >= 16 + 2 * mw) x.list[e - 16 - 2 * mw] = v;
      else if (e >= 16) x.sel[(e - 16) / mw][(e - 16) % mw] = (uint32_t)v;
      else if (e == 0) x.n_union = v;
      else if (e == 1) x.n_cent = v;
      else if (e == 2) x.present[1] = v;
      else if (e >= 4 && e < 12) x.cent[e - 4] = v;
    }
    if (tid == 0) x.present[0] = 1;
  }
  cta_sync();
#ifdef SOL_TRACE
  if (tid == 0) SOL_GT_AT(9);
#endif
#ifdef SOL_TRACE
  if (tid == 0) SOL_GT_AT(10);
#endif
  // Centroid offsets (log2 units; -inf where the half took the block exactly
  // or past the last block) and, per 64-column half, whether any is live:
  // warp w takes the (tile, query half) pairs w, w + 12, ...
  for (int pr = warp; pr < 2 * x.n_cent; pr += kThreads / 32) {
    const int slot = pr >> 1, hf = pr & 1;
    bool l0 = false, l1 = false;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = lane + 32 * q, j = 128 * x.cent[slot] + c;
      const bool live = x.present[hf] && j < a.nkb && !((x.sel[hf][j >> 5] >> (j & 31)) & 1u);
      if (!I8) x.cent_add[slot][hf][c] = live ? x.cbias[j] * kLog2e : -INFINITY;
      if (q < 2) l0 |= live; else l1 |= live;
    }
    const bool any0 = __any_sync(0xffffffffu, l0), any1 = __any_sync(0xffffffffu, l1);
    if (lane == 0) { x.cent_live[slot][hf][0] = any0; x.cent_live[slot][hf][1] = any1; }
  }
  fence_before();
  cta_sync();
  fence_after();
  const uint32_t tmem = x.tmem_base;
#ifdef SOL_TRACE
  if (tid == 0 && SOL_TRACE_ON) { x.trace[9 * kTraceSteps] = t_entry; x.trace[9 * kTraceSteps + 8] = g_entry; SOL_TRACE_AT(10, 0); SOL_GT_AT(1); }
#endif
  const int n_ex = (x.n_union + 1) >> 1;
  const int T = n_ex + x.n_cent;

  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(kRegsControl));
  if (warp == kKWarp || warp == kVWarp) {
    // ---------------------------------------------------------------- TMA producers
    // Q and the K tiles (kKStages ring) from one warp, the V tiles (kVStages
    // ring) from another; each runs ahead on its own ring.
    if (lane == 0) {
      const bool is_k = warp == kKWarp;
      const int nst = is_k ? kKStages : kVStages;
      const CUtensorMap* m4 = is_k ? &mk : &mv;
      const CUtensorMap* m3 = is_k ? &mkb : &mvb;
      uint8_t* ring = is_k ? sK : sV;
      int nl = 0;   // tile loads issued
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % nst, n = t / nst;
        int j0 = 0, j1 = 0, ct = -1;
        if (t < n_ex) {
          j0 = x.list[2 * t] & 0xffff;
          j1 = (2 * t + 1 < x.n_union) ? (x.list[2 * t + 1] & 0xffff) : j0;
        } else {
          ct = x.cent[t - n_ex];
        }
        // K stage t%3 is free once QK(t-3) is complete (the completion of
        // s_full[t%3] before the one for S(t)); V stage t%2 once PV(t-2) is
        // (o_done[t%2]): the same commits that signal the consumers.
        uint64_t* empty = is_k ? &bar.s_full[s] : &bar.o_done[s];
        uint64_t* full = is_k ? &bar.k_full[s] : &bar.v_full[s];
        if (!(ok = wait_bar(empty, (n & 1) ^ 1, abort_flag, a.status))) break;
        // INT8: the stage's block means of step t-3 must also have been read by the softmax
        if (I8 && is_k && !(ok = wait_bar(&bar.kb_done[s], (n & 1) ^ 1, abort_flag, a.status))) break;
        SOL_TRACE_AT(is_k ? 7 : 8, t);
        uint8_t* dst = ring + s * C::kTileBytes;
        ++nl;
        if (I8 && is_k && ct < 0) {
          // residual codes of the two key blocks (64 rows x 128 bytes each) and their bf16 means
          mbar_expect_tx(full, C::kK8Bytes + 2 * D * 2);
          tma_load_3d(dst, &mk8, 0, 64 * j0, (int)bh, full);
          tma_load_3d(dst + C::kK8Bytes / 2, &mk8, 0, 64 * j1, (int)bh, full);
          bulk_load(dst + C::kKMeanOff, a.kmean16 + ((int64_t)bh * a.nkb + j0) * D, D * 2, full);
          bulk_load(dst + C::kKMeanOff + D * 2, a.kmean16 + ((int64_t)bh * a.nkb + j1) * D, D * 2, full);
        } else {
          mbar_expect_tx(full, C::kTileBytes);
          for (int c = 0; c < C::kChunks; ++c) {
            if (ct < 0) {
              tma_load_4d(dst + c * C::kChunkBytes, m4, c * 64, h, 64 * j0, b, full);
              tma_load_4d(dst + c * C::kChunkBytes + C::kChunkBytes / 2, m4, c * 64, h, 64 * j1, b, full);
            } else {
              tma_load_3d(dst + c * C::kChunkBytes, m3, c * 64, 128 * ct, (int)bh, full);
            }
          }
        }
      }
      // drain: every armed load has landed before the CTA may exit
      for (int s = 0; s < nst; ++s) {
        const int cnt = (nl + nst - 1 - s) / nst;
        if (cnt) drain_bar(is_k ? &bar.k_full[s] : &bar.v_full[s], (cnt - 1) & 1, a.status);
      }
      if (is_k) drain_bar(&bar.q_full, 0, a.status);
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    // Issue order QK(0), QK(1), QK(2), PV(0), QK(3), PV(1), QK(4), ...  Step t
    // uses S_(t%3), whose first 64 columns the softmax overwrites with P(t);
    // every PV accumulates into the one O.  QK(t+3) follows PV(t) in the
    // (in-order) tensor pipe, so it overwrites S_(t%3) only after PV(t) has
    // read P(t), and the commit that signals S(t+3) also covers PV(t).
    {   // the whole warp runs the loop; one elected lane issues each MMA / commit
      // The tensor pipe's issue queue is short, so the steady-state loop is
      // kept free of run-time conditions around its MMA batches (a batch
      // under a condition costs pipe time even when skipped): the first PV
      // (which starts O) and the last three (no QK follows) are peeled off,
      // ring positions are counters, descriptors are precomputed (one add
      // per MMA) and every wait sits between batches.
      constexpr uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t id_pv = idesc_bf16(128, D, 0, 1);
      constexpr int NQ = D / 16;                                   // QK MMAs (k = 16 each)
      constexpr uint64_t kStageD = (uint64_t)(C::kTileBytes >> 4); // descriptor step per ring stage
      const uint64_t qd = sdesc(smem_u32(sQ), 16, 1024);
      const uint64_t kd0 = sdesc(smem_u32(sK), 16, 1024);
      const uint64_t vd0 = sdesc(smem_u32(sV), C::kChunkBytes, 1024);
      int kst = 0, vst = 0, sq = 0, sp = 0;        // K / V ring stages, S buffers of the next QK / PV
      uint32_t kph = 0, vph = 0, pph = 0;          // their phase parities
      // QK(g) into S_sq from K stage kst (K must have landed); with INT8 QK the exact
      // tiles (the first n_ex) run s8 x s8 -> s32 on the query and residual key codes
      // (K = 32 bytes per MMA, one 128-byte chunk per row), the centroid tiles bf16
      int nqk = 0;
      auto qk = [&]() {
        const uint64_t kd = kd0 + (uint64_t)kst * kStageD;
        const uint32_t d = tmem + 128 * sq;
        if (I8 && nqk < n_ex) {
          constexpr uint32_t id_qk8 = idesc_s8(128, 128);
          const uint64_t q8d = sdesc(smem_u32(sQ8), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_ss_i8_w(d, q8d + (uint64_t)(kk * 2), kd + (uint64_t)(kk * 2), id_qk8, kk > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < NQ; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * C::kChunkBytes + (kk & 3) * 32) >> 4);
            mma_ss_w(d, qd + off, kd + off, id_qk, kk > 0 ? 1u : 0u);
          }
        }
        ++nqk;
        mma_commit_w(&bar.s_full[sq]);   // also frees K stage kst (== sq)
        if (++kst == kKStages) { kst = 0; kph ^= 1u; }
        sq = sq == 2 ? 0 : sq + 1;
      };
      // PV(u) from P in S_sp and V stage vst into O (P and V must be ready)
      auto pv = [&](int u, bool first) {
        const uint64_t vd = vd0 + (uint64_t)vst * kStageD;
        const uint32_t pa = tmem + 128 * sp;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_w(tmem + kOCol, pa + kk * 8, vd + (uint64_t)(kk * 2048 >> 4), id_pv, (first && kk == 0) ? 0u : 1u);
        mma_commit_w(&bar.o_done[u & 1]);   // also frees V stage vst (== u % 2)
        if (++vst == kVStages) { vst = 0; vph ^= 1u; }
        if (sp == 2) { sp = 0; pph ^= 1u; } else { ++sp; }
      };
      // every wait's outcome is made warp-uniform, so all lanes leave the loop together
      auto wait_k = [&]() {   // TMA data: the mbarrier completion orders it, no tcgen05 fence needed
        return __all_sync(0xffffffffu, wait_bar(&bar.k_full[kst], kph, abort_flag, a.status));
      };
      auto wait_pv = [&]() {
        const bool r = __all_sync(0xffffffffu, wait_bar(&bar.p_full[sp], pph, abort_flag, a.status) &&
                                                   wait_bar(&bar.v_full[vst], vph, abort_flag, a.status));
        fence_after();
        return r;
      };
      bool ok = __all_sync(0xffffffffu, wait_bar(&bar.q_full, 0, abort_flag, a.status));
      if (I8 && ok) {   // the softmax quantizes the query tile first
        ok = __all_sync(0xffffffffu, wait_bar(&bar.q8_ready, 0, abort_flag, a.status));
        fence_after();
      }
      const int nq0 = T < 3 ? T : 3;
      for (int g = 0; g < nq0 && ok; ++g) {
        if ((ok = wait_k())) qk();
      }
      const int n_steady = T > 3 ? T - 3 : 0;    // PV(u) followed by QK(u+3)
      if (ok && T > 0 && (ok = wait_pv())) {
        SOL_TRACE_AT(5, 0);
        pv(0, true);
        if (n_steady > 0 && (ok = wait_k())) qk();
      }
      for (int u = 1; u < n_steady && ok; ++u) {
        if (!(ok = wait_pv())) break;
        SOL_TRACE_AT(5, u);
        pv(u, false);
        SOL_TRACE_AT(13, u);
        if (!(ok = wait_k())) break;
        SOL_TRACE_AT(4, u + 3);
        qk();
        SOL_TRACE_AT(11, u + 3);
      }
      for (int u = n_steady > 1 ? n_steady : 1; u < T && ok; ++u) {
        if (!(ok = wait_pv())) break;
        pv(u, false);
      }
      // all issued MMAs complete before the epilogue reads O and TMEM is released
      mma_commit_w(&bar.final_mma);
      drain_bar(&bar.final_mma, 0, a.status);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(kRegsSoftmax));
    // ---------------------------------------------------------------- softmax warpgroups
    // Warpgroup w (warps 4w+4 .. 4w+7) takes the steps t = w, w+3, w+6, ...,
    // i.e. always S buffer w, one thread per row (TMEM lane), so the three
    // groups' TMEM loads, exponentials and waits overlap.  All feed the one
    // accumulator O, so they share each row's reference max m (log2 units):
    // step t reads the reference left by step t-1 (the previous group),
    // raises it only when its tile's max exceeds it by more than 2^8 (lazy
    // rescaling), publishes it at once and then exponentiates against it.
    // A raise rescales O after PV(t-1), the last product taken against the
    // old reference.  Each group keeps its partial sum l_w relative to the
    // reference of its latest step; the epilogue brings all to the final
    // reference.  A thread holds half an S row at a time (the register
    // budget of three groups), so the row max reads S once and the
    // exponentials read it again.
    const int w = (warp >> 2) - 1;            // softmax warpgroup 0 .. kSoftmaxGroups-1
    const int sub = warp & 3;                 // TMEM sub-partition = rows 32*sub .. 32*sub+31
    const int r = 32 * sub + lane;            // row of the tile
    const int hf = r >> 6;                    // query block half (warp-uniform)
    const bool present = x.present[hf] != 0;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * sub) << 16);
    const uint32_t o_addr = lane_addr + kOCol;
    const float sl2 = a.scale * kLog2e;
#ifndef SOL_TRACE_WARP
#define SOL_TRACE_WARP 0
#endif
    const bool tracer = sub == SOL_TRACE_WARP && lane == 0;
    (void)tracer;
    float ref_w = -INFINITY, l = 0.f;         // this group's partial sum, relative to ref_w
    bool ok = true;
    const int bb = w;                         // S buffer of every step of this group: t % 3 = w
    static_assert(kSoftmaxGroups == 3, "one softmax warpgroup per S buffer");
    float sigq = 0.f;                         // INT8 QK: this row's query scale
    if constexpr (I8) {
      // Quantize the query tile once: every softmax thread takes its row's max |q| (exact
      // on bf16 values), sigma_q = max / 127, and writes the codes rint(q * (1 / sigma_q))
      // of the 16-byte code units u = w, w + 3, ... of its row into the SW128 code tile.
      ok = __all_sync(0xffffffffu, wait_bar(&bar.q_full, 0, abort_flag, a.status));
      float amax = 0.f;
      if (ok) {
        for (int c = 0; c < C::kChunks; ++c) {
#pragma unroll
          for (int pu = 0; pu < 8; ++pu) {
            float f[8];
            bf16x8_f32(*reinterpret_cast<const uint4*>(sQ + c * C::kChunkBytes + r * 128 + pu * 16), f);
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
          }
        }
      }
      const float sg = amax / 127.f;
      const float inv = sg > 0.f ? 1.f / sg : 0.f;
      if (ok) {
        for (int u = w; u < D / 16; u += kSoftmaxGroups) {   // code unit u: dims 16u .. 16u+15
          const int c = u >> 2, lu0 = 2 * (u & 3);           // its 64-dim chunk, first bf16 unit there
          float f[16];
          bf16x8_f32(*reinterpret_cast<const uint4*>(sQ + c * C::kChunkBytes + r * 128 + ((lu0 ^ (r & 7)) << 4)), f);
          bf16x8_f32(*reinterpret_cast<const uint4*>(sQ + c * C::kChunkBytes + r * 128 + (((lu0 + 1) ^ (r & 7)) << 4)),
                     f + 8);
          uint32_t wd[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t word = 0u;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int qc = sg > 0.f ? min(127, max(-127, __float2int_rn(__fmul_rn(f[4 * q4 + i], inv)))) : 0;
              word |= (uint32_t)(qc & 0xff) << (8 * i);
            }
            wd[q4] = word;
          }
          *reinterpret_cast<uint4*>(sQ8 + r * 128 + ((u ^ (r & 7)) << 4)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
      }
      if (w == 0) x.qsig[r] = sg;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the codes feed the tensor cores
      mbar_arrive(&bar.q8_ready);
      if (ok) ok = __all_sync(0xffffffffu, wait_bar(&bar.q8_ready, 0, abort_flag, a.status));
      sigq = x.qsig[r];
    }
    for (int t = w; t < T && ok; t += kSoftmaxGroups) {
#ifdef SOL_TRACE
      if (tracer) SOL_TRACE_AT(15, t);
#endif
      // which 64-column halves of this S tile the row uses, and their additive offsets
      bool need0, need1;
      const float *add0 = nullptr, *add1 = nullptr;
      const int slot = t - n_ex;                // centroid tiles: their slot
      int j0 = 0, j1 = 0;                       // exact tiles: the two key blocks
      if (t < n_ex) {
        const int e0 = x.list[2 * t];
        const int e1 = (2 * t + 1 < x.n_union) ? x.list[2 * t + 1] : -1;
        j0 = e0 & 0xffff;
        j1 = e1 >= 0 ? (e1 & 0xffff) : j0;
        need0 = present && ((e0 >> (16 + hf)) & 1);
        need1 = present && e1 >= 0 && ((e1 >> (16 + hf)) & 1);
        add0 = (j0 == a.nkb - 1) ? x.tail_add : nullptr;
        add1 = (e1 >= 0 && j1 == a.nkb - 1) ? x.tail_add : nullptr;
      } else {
        need0 = x.cent_live[slot][hf][0] != 0;
        need1 = x.cent_live[slot][hf][1] != 0;
        if (!I8) {
          add0 = x.cent_add[slot][hf];
          add1 = x.cent_add[slot][hf] + 64;
        }
      }
      // INT8 exact tile: each half's logit is cc * S_int + mm (log2 units), with
      // cc = s log2(e) sigma_q sigma_j and mm = s log2(e) q . kmean16_j, the mean term
      // computed here, before S is ready, from the stage's bf16 block means
      float cc0 = 0.f, cc1 = 0.f, mm0 = 0.f, mm1 = 0.f;
      if constexpr (I8) {
        // Every step, centroid tiles included, waits for its stage's load before it
        // releases the stage: the producer has then passed its wait for this step, so
        // the kb_done phases never run two ahead of it (its parity wait could not tell
        // the phase it waits for from the one after next).
        const int ks = t % kKStages;
        ok = __all_sync(0xffffffffu, wait_bar(&bar.k_full[ks], (t / kKStages) & 1, abort_flag, a.status));
        if (!ok) break;
        if (t < n_ex) {
          if (need0 || need1) {
            const uint8_t* km = sK + ks * C::kTileBytes + C::kKMeanOff;
            // packed f32x2 FMAs over dim pairs: two interleaved partial sums per block
            uint64_t a0 = 0ull, a1 = 0ull;
            auto pair = [](uint32_t w) { return f2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)); };
#pragma unroll 4
            for (int u = 0; u < D / 8; ++u) {   // 8 dims per 16-byte unit
              const int c = u >> 3, lu = u & 7;
              const uint4 qv = *reinterpret_cast<const uint4*>(sQ + c * C::kChunkBytes + r * 128 + ((lu ^ (r & 7)) << 4));
              const uint4 k0 = *reinterpret_cast<const uint4*>(km + u * 16);
              const uint4 k1 = *reinterpret_cast<const uint4*>(km + D * 2 + u * 16);
              const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w}, k0w[4] = {k0.x, k0.y, k0.z, k0.w},
                             k1w[4] = {k1.x, k1.y, k1.z, k1.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const uint64_t q2 = pair(qw[e]);
                a0 = ffma2(q2, pair(k0w[e]), a0);
                a1 = ffma2(q2, pair(k1w[e]), a1);
              }
            }
            float d0, d1, lo, hi;
            f2unpack(a0, lo, hi);
            d0 = lo + hi;
            f2unpack(a1, lo, hi);
            d1 = lo + hi;
            const float sq = sl2 * sigq;
            cc0 = sq * __ldg(a.ksig + bh * a.nkb + j0);
            cc1 = sq * __ldg(a.ksig + bh * a.nkb + j1);
            mm0 = sl2 * d0;
            mm1 = sl2 * d1;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.kb_done[ks]);   // the stage may be reloaded (after QK(t) too)
      }
      ok = __all_sync(0xffffffffu, wait_bar(&bar.s_full[bb], (t / 3) & 1, abort_flag, a.status));
      if (!ok) break;
      fence_after();
#ifdef SOL_TRACE
      if (tracer) SOL_TRACE_AT(0, t);
      if (lane == 0) SOL_TRACE_AT(20 + sub, t);
#endif
      const uint32_t s_addr = lane_addr + 128 * bb;   // S(t); P(t) is written over its first 64 columns
      const bool i8x = I8 && t < n_ex;                // this S tile holds s32 INT8 products
      const bool i8c = I8 && t >= n_ex;               // INT8 variant, centroid tile: offsets computed here
      // centroid-column offsets of columns col .. col+3 of half hh (INT8 variant: no table)
      auto coff4 = [&](int hh, int col) {
        const int j = 128 * x.cent[slot < 0 ? 0 : slot] + 64 * hh + col;
        const float4 cb = *reinterpret_cast<const float4*>(&x.cbias[j]);
        const uint32_t bits = x.sel[hf][j >> 5] >> (j & 31);
        const bool pr = present;
        float4 o;
        o.x = (pr && j + 0 < a.nkb && !(bits & 1u)) ? cb.x * kLog2e : -INFINITY;
        o.y = (pr && j + 1 < a.nkb && !(bits & 2u)) ? cb.y * kLog2e : -INFINITY;
        o.z = (pr && j + 2 < a.nkb && !(bits & 4u)) ? cb.z * kLog2e : -INFINITY;
        o.w = (pr && j + 3 < a.nkb && !(bits & 8u)) ? cb.w * kLog2e : -INFINITY;
        return o;
      };
      // pass 1: the tile's row max (log2 units), one 64-column half at a time;
      // pass 2 below reloads each half for its exponentials (the register
      // budget of three softmax warpgroups holds half a row, not a whole one)
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (!(hh ? need1 : need0)) continue;
        const float* ad = hh ? add1 : add0;
        float v[64];
        tmem_ld32(s_addr + 64 * hh, v);
        tmem_ld32(s_addr + 64 * hh + 32, v + 32);
        tmem_wait_ld();
        if (i8x) {
          const float cc = hh ? cc1 : cc0, mm = hh ? mm1 : mm0;
          if (ad) {   // the tail block: per column, with its -inf past N
#pragma unroll
            for (int c = 0; c < 64; ++c) m4[c & 3] = fmaxf(m4[c & 3], fmaf(i2f_exact(v[c]), cc, mm) + ad[c]);
          } else {    // cc >= 0: the largest code product gives the largest logit
            int im = INT_MIN;
#pragma unroll
            for (int c = 0; c < 64; ++c) im = max(im, __float_as_int(v[c]));
            m4[0] = fmaxf(m4[0], fmaf((float)im, cc, mm));
          }
        } else if (ad || i8c) {
          const uint64_t sl22 = f2pack(sl2, sl2);
          const float4* ad4 = reinterpret_cast<const float4*>(ad);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float4 o = i8c ? coff4(hh, 4 * c) : ad4[c];
            f2unpack(ffma2(f2pack(v[4 * c], v[4 * c + 1]), sl22, f2pack(o.x, o.y)), v[4 * c], v[4 * c + 1]);
            f2unpack(ffma2(f2pack(v[4 * c + 2], v[4 * c + 3]), sl22, f2pack(o.z, o.w)), v[4 * c + 2], v[4 * c + 3]);
            m4[c & 3] = fmax3(m4[c & 3], v[4 * c], v[4 * c + 1]);
            m4[(c + 2) & 3] = fmax3(m4[(c + 2) & 3], v[4 * c + 2], v[4 * c + 3]);
          }
        } else {
          float r4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 32; ++c) r4[c & 3] = fmax3(r4[c & 3], v[2 * c], v[2 * c + 1]);
#pragma unroll
          for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], r4[q] * sl2);
        }
      }
      const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
#ifdef SOL_TRACE
      if (tracer) SOL_TRACE_AT(1, t);
#endif
      // the reference after step t-1, raised if this tile exceeds it by more than 2^8
      float m_prev = -INFINITY;
      if (t > 0) {
        ok = __all_sync(0xffffffffu, wait_bar(&bar.ref_full[(w + kSoftmaxGroups - 1) % kSoftmaxGroups][sub],
                                              ((t - 1) / kSoftmaxGroups) & 1, abort_flag, a.status));
        if (!ok) break;
        m_prev = x.m_ref[r];
      }
#ifdef SOL_TRACE
      if (tracer) SOL_TRACE_AT(6, t);
#endif
      float m_cur = m_prev;
      if (mt > m_prev + kRescale || (m_prev == -INFINITY && mt != -INFINITY)) m_cur = mt;
      x.m_ref[r] = m_cur;
      mbar_arrive(&bar.ref_full[w][sub]);
      const bool resc = m_cur != m_prev && m_prev != -INFINITY;   // O holds terms against m_prev
      if (m_cur != ref_w) { l *= ex2(ref_w - m_cur); ref_w = m_cur; }   // m only grows: ex2(<= 0)
      const float base = (m_cur == -INFINITY) ? 0.f : m_cur;
      // p = 2^(x - base) as bf16 pairs into P(t) (over S(t)'s first 64 columns)
      float lsum = 0.f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t pk[32];
        if (hh ? need1 : need0) {
          const float* ad = hh ? add1 : add0;
          float v[64];
          tmem_ld32(s_addr + 64 * hh, v);
          tmem_ld32(s_addr + 64 * hh + 32, v + 32);
          tmem_wait_ld();
          uint64_t mul2, nb2;
          if (i8x) {   // s32 products: exact float, then cc * S + mm (+ tail offset) - base
            const float cc = hh ? cc1 : cc0, mm = hh ? mm1 : mm0;
            const uint64_t cc2 = f2pack(cc, cc), mb2 = f2pack(mm - base, mm - base);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              f2unpack(ffma2(f2pack(i2f_exact(v[2 * c]), i2f_exact(v[2 * c + 1])), cc2, mb2), v[2 * c], v[2 * c + 1]);
              if (ad) { v[2 * c] += ad[2 * c]; v[2 * c + 1] += ad[2 * c + 1]; }
            }
            mul2 = f2pack(1.f, 1.f);
            nb2 = 0ull;   // packed (0, 0): base already taken off
          } else {
            if (ad || i8c) {   // offset logits in log2 units, as in pass 1
              const uint64_t sl22 = f2pack(sl2, sl2);
              const float2* ad2 = reinterpret_cast<const float2*>(ad);
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                float2 o;
                if (i8c) {
                  const float4 o4 = coff4(hh, 4 * (c >> 1));
                  o = (c & 1) ? make_float2(o4.z, o4.w) : make_float2(o4.x, o4.y);
                } else {
                  o = ad2[c];
                }
                f2unpack(ffma2(f2pack(v[2 * c], v[2 * c + 1]), sl22, f2pack(o.x, o.y)), v[2 * c], v[2 * c + 1]);
              }
            }
            const float mul = (ad != nullptr || i8c) ? 1.f : sl2;   // offset logits are in log2 units
            mul2 = f2pack(mul, mul);
            nb2 = f2pack(-base, -base);
          }
          uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float x0, x1;
            f2unpack(ffma2(f2pack(v[2 * c], v[2 * c + 1]), mul2, nb2), x0, x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            acc2[c & 1] = fadd2(acc2[c & 1], f2pack(p0, p1));
            pk[c] = pack_bf16(p0, p1);
          }
          float a0, a1, a2, a3;
          f2unpack(acc2[0], a0, a1);
          f2unpack(acc2[1], a2, a3);
          lsum += (a0 + a1) + (a2 + a3);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = 0u;
        }
        tmem_st32(s_addr + 32 * hh, pk);
      }
      l += lsum;
#ifdef SOL_TRACE
      if (tracer) SOL_TRACE_AT(2, t);
#endif
      if (__any_sync(0xffffffffu, resc)) {
        // O = sum of PV(0..t-1) against m_prev once PV(t-1) is complete
        ok = __all_sync(0xffffffffu,
                        wait_bar(&bar.o_done[(t - 1) & 1], ((t - 1) >> 1) & 1, abort_flag, a.status));
        if (!ok) break;
        fence_after();
        rescale_rows<D>(o_addr, resc ? ex2(m_prev - m_cur) : 1.f);
      }
      tmem_wait_st();
      fence_before();
      __syncwarp();
#ifdef SOL_TRACE
      if (tracer) SOL_TRACE_AT(3, t);
      if (lane == 0) SOL_TRACE_AT(16 + sub, t);
#endif
#ifdef SOL_FAULT_TEST
      // fault-test build: the arrive of step g_drop_p_arrive is withheld, so the
      // MMA warp's bounded wait for P(t) expires (sol_debug_drop_arrive)
      if (lane == 0 && t != g_drop_p_arrive) mbar_arrive(&bar.p_full[bb]);
#else
      if (lane == 0) mbar_arrive(&bar.p_full[bb]);
#endif
    }
    // epilogue: with M the final reference, O / (l_0 2^(ref_0 - M) + l_1 2^(ref_1 - M));
    // warpgroup w writes the columns [w D/2, (w+1) D/2)
#ifdef SOL_TRACE
    if (tracer && w < 2) { SOL_TRACE_AT(12, w); SOL_GT_AT(2 + w); }
#endif
    x.ml[w][r] = make_float2(ref_w, l);
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(&bar.final_mma, 0, abort_flag, a.status));
    named_bar_sync(1, 128 * kSoftmaxGroups);
    if (ok && !*abort_flag && T > 0) {
      fence_after();
      const float M = x.m_ref[r];            // written by step T-1
      float L = 0.f;
#pragma unroll
      for (int g = 0; g < kSoftmaxGroups; ++g) {
        const float2 pg = x.ml[g][r];
        if (pg.x != -INFINITY) L += pg.y * ex2(pg.x - M);
      }
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const int grow = 64 * (i0 + hf) + (r & 63);
      const bool store = present && grow < a.N;
      __nv_bfloat16* orow = a.o + (int64_t)b * a.ob + (int64_t)h * a.oh + (int64_t)grow * a.on;
      for (int c = w; c < D / 32; c += kSoftmaxGroups) {   // 32-column chunks, dealt round the groups
        const int col = 32 * c;
        float ov[32];
        tmem_ld32(o_addr + col, ov);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            const uint4 u4 = make_uint4(pack_bf16(ov[e] * inv, ov[e + 1] * inv), pack_bf16(ov[e + 2] * inv, ov[e + 3] * inv),
                                        pack_bf16(ov[e + 4] * inv, ov[e + 5] * inv), pack_bf16(ov[e + 6] * inv, ov[e + 7] * inv));
            *reinterpret_cast<uint4*>(orow + col + e) = u4;
          }
        }
      }
      if (w == 0 && store && a.lse) a.lse[bh * a.N + grow] = (M + log2f(L)) * kLn2;
    }
  }
#ifdef SOL_TRACE
  if (warp >= 4 && warp < 12 && (warp & 3) == SOL_TRACE_WARP && lane == 0) { SOL_TRACE_AT(14, (warp >> 2) - 1); SOL_GT_AT(4 + (warp >> 2) - 1); }
#endif
  fence_before();
  cta_sync();
#ifdef SOL_TRACE
  if (tid == 0) { SOL_TRACE_AT(9, 1); SOL_GT_AT(6); }
  if (warp == kMmaWarp && lane == 0) SOL_GT_AT(7);
  cta_sync();
  if (SOL_TRACE_ON)
    for (int i = tid; i < kTraceSlots * kTraceSteps; i += kThreads) g_trace[i] = x.trace[i];
#endif
  if (warp == kMmaWarp) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(512));
  }
}

// ---- host side: tensor maps and launch ------------------------------------------------------------
static_assert(1024 + Cfg<128, false>::kSmemTiles + sizeof(Extra<false>) <= 232448, "bf16 variant: shared memory");
static_assert(1024 + Cfg<128, true>::kSmemTiles + sizeof(Extra<true>) <= 232448, "INT8 variant: shared memory");

template <int D, bool I8>
cudaError_t launch_tc(const AttnArgs& a, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mkb, mvb, mk8;
  const cuuint64_t bstride = (cuuint64_t)(a.B > 1 ? a.sb : (int64_t)a.N * a.sn) * 2;
  const cuuint64_t dims4[4] = {(cuuint64_t)D, (cuuint64_t)a.H, (cuuint64_t)a.N, (cuuint64_t)a.B};
  const cuuint64_t str4[3] = {(cuuint64_t)a.sh * 2, (cuuint64_t)a.sn * 2, bstride};
  const cuuint32_t box4[4] = {64, 1, 64, 1};
  const cuuint64_t dims3[3] = {(cuuint64_t)D, (cuuint64_t)a.nkb, (cuuint64_t)a.B * a.H};
  const cuuint64_t str3[2] = {(cuuint64_t)D * 2, (cuuint64_t)a.nkb * D * 2};
  const cuuint32_t box3[3] = {64, 128, 1};
  if (!make_map(&mq, a.q, 4, dims4, str4, box4, kSw128) || !make_map(&mk, a.k, 4, dims4, str4, box4, kSw128) ||
      !make_map(&mv, a.v, 4, dims4, str4, box4, kSw128) || !make_map(&mkb, a.kbar16, 3, dims3, str3, box3, kSw128) ||
      !make_map(&mvb, a.vbar16, 3, dims3, str3, box3, kSw128))
    return cudaErrorInvalidValue;
  mk8 = mk;   // unused by the bf16 variant
  if (I8) {   // residual key codes, head-major [B*H, N, D] bytes: 64-row boxes of 128-byte rows
    const cuuint64_t dims8[3] = {(cuuint64_t)D, (cuuint64_t)a.N, (cuuint64_t)a.B * a.H};
    const cuuint64_t str8[2] = {(cuuint64_t)D, (cuuint64_t)a.N * D};
    const cuuint32_t box8[3] = {(cuuint32_t)D, 64, 1};
    if (!make_map(&mk8, a.kcode, 3, dims8, str8, box8, kSw128, CU_TENSOR_MAP_DATA_TYPE_UINT8))
      return cudaErrorInvalidValue;
  }
  TcParams prm{a, (a.nkb + 31) / 32};
  const int64_t tiles = (int64_t)a.B * a.H * ((a.nqb + 1) / 2);
  plan_kernel<<<(unsigned)((tiles + kPlanWarps - 1) / kPlanWarps), kPlanWarps * 32, 0, st>>>(a, prm.mask_words);
  cudaError_t pe = cudaGetLastError();
  if (pe != cudaSuccess) return pe;
  const size_t smem = 1024 + Cfg<D, I8>::kSmemTiles + sizeof(Extra<I8>);
  // Once per device (so that launches stay free of attribute calls, e.g.
  // inside a stream capture): opt in to the shared memory, and check the
  // register count.  The setmaxnreg split is sized for exactly kRegsLaunch
  // registers per thread at launch; with any other count the softmax
  // warpgroups' increase could not be granted, so refuse to launch.
  static std::atomic<int> prepared[64];   // zero-initialised; set once per device (any thread)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !prepared[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(attn_tc_kernel<D, I8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, attn_tc_kernel<D, I8>)) != cudaSuccess) return e;
    if (fa.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < 64) prepared[dev].store(1, std::memory_order_release);
  }
  dim3 grid((a.nqb + 1) / 2, a.H, a.B);
  attn_tc_kernel<D, I8><<<grid, kThreads, smem, st>>>(mq, mk, mv, mkb, mvb, mk8, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn(const AttnArgs& a, int D, cudaStream_t st) {
  if (a.qk_int8) return D == 128 ? launch_tc<128, true>(a, st) : cudaErrorInvalidValue;
  return D == 128 ? launch_tc<128, false>(a, st) : launch_tc<64, false>(a, st);
}

#ifdef SOL_FAULT_TEST
cudaError_t set_drop_p_arrive(int step) {
  return cudaMemcpyToSymbol(g_drop_p_arrive, &step, sizeof(int));
}
#endif

}  // namespace sol

#ifdef SOL_TRACE
// Copies the phase trace (24 slots x 128 steps of 32-bit clock stamps) to host memory.
extern "C" int sol_debug_trace(unsigned int* host, int n) {
  const int total = sol::kTraceSlots * sol::kTraceSteps;
  return (int)cudaMemcpyFromSymbol(host, sol::g_trace, sizeof(unsigned int) * (n < total ? n : total));
}
#endif
