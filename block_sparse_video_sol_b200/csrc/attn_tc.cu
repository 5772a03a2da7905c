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
// Roles (7 warps):
//   warp 0     TMA producer: Q once, then the K tiles into a 3-stage ring.
//   warp 6     TMA producer: the V tiles into a 2-stage ring.
//   warp 1     MMA issuer (one lane): S_b = Q K^T into TMEM buffer b = t%2,
//              then O += P V with P read from its own TMEM buffer.
//   warps 2-5  softmax, one thread per row (TMEM lane): online max/sum in
//              fp32 with lazy rescaling (O in TMEM is rescaled only when a
//              row's max grows by more than 2^8), P written back to TMEM,
//              final normalisation and bf16 store.
// TMEM: S0 = columns [0,128), S1 = [128,256), O = [256, 256+D),
//       P0 = [384, 448), P1 = [448, 512) (bf16 pairs).
// Every mbarrier wait is bounded; on expiry the kernel raises
// SOL_ERR_TIMEOUT, stops issuing, drains what it issued and frees TMEM.
#include <cuda.h>
#include <math.h>

#include "common.cuh"

namespace sol {
namespace {

constexpr int kThreads = 224;
constexpr int kKStages = 3;   // K tiles in flight (needed first, by QK)
constexpr int kVStages = 2;   // V tiles in flight (needed a softmax later, by PV)

// Optional phase trace (build with -DSOL_TRACE): clock64() stamps of one CTA's
// roles for its first kTraceSteps S tiles, read back with sol_debug_trace().
#ifdef SOL_TRACE
constexpr int kTraceSteps = 256;
__device__ long long g_trace[16 * kTraceSteps];
#define SOL_TRACE_AT(slot, step) \
  do { if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && (step) < kTraceSteps) \
         g_trace[(slot) * kTraceSteps + (step)] = clock64(); } while (0)
#else
#define SOL_TRACE_AT(slot, step) do { } while (0)
#endif
constexpr uint32_t kSpinLimit = 1u << 22;
constexpr float kRescale = 8.0f;   // log2 units: rescale O when the max grows by more than 2^8
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxWords = kMaxKeyBlocks / 32;
constexpr int kMaxCentTiles = kMaxKeyBlocks / 128;

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;               // 128-byte column chunks per row
  static constexpr int kChunkBytes = 128 * 128;        // one chunk of a 128-row tile
  static constexpr int kTileBytes = 128 * D * 2;       // Q, K or V tile of 128 rows
  static constexpr int kSmemTiles = kTileBytes * (1 + kKStages + kVStages);
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], s_free[2], p_full[2], o_done[2], final_mma;
};

struct Extra {
  Bars bar;
  uint32_t tmem_base;
  int abort_flag;
  int n_union, n_cent, present[2];
  uint32_t sel[2][kMaxWords];        // exact-block bitmaps of the two halves
  int cent[kMaxCentTiles];           // centroid tiles to visit
  int list[kMaxKeyBlocks];           // union entries: j | needA << 16 | needB << 17
  int cent_live[kMaxCentTiles][2][2];           // [slot][half][64-column half]: any live centroid
  float cent_add[kMaxCentTiles][2][128];        // log2-unit offset of each centroid column, -inf if masked
  float tail_add[64];                           // 0 for valid rows of the last key block, -inf beyond N
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t c) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(b)), "r"(c));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
               : "=r"(ok) : "r"(smem_u32(b)), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait: false (and the CTA-wide abort flag set) on expiry or abort.
__device__ __forceinline__ bool wait_bar(uint64_t* b, uint32_t parity, volatile int* abort_flag, int* status) {
  for (uint32_t i = 0;; ++i) {
    if (mbar_try(b, parity)) return true;
    if (*abort_flag) return false;
    if (i >= kSpinLimit) {
      *abort_flag = 1;
      raise_status(status, SOL_ERR_TIMEOUT);
      return false;
    }
    if (i > 2048) __nanosleep(64);
  }
}

// Bounded wait that ignores the abort flag: used to drain issued copies / MMAs
// before the CTA releases shared memory and TMEM.
__device__ __forceinline__ void drain_bar(uint64_t* b, uint32_t parity, int* status) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try(b, parity)) return;
    if (i > 32) __nanosleep(64);
  }
  raise_status(status, SOL_ERR_TIMEOUT);
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* m, int c0, int c1, int c2, int c3, uint64_t* bar) {
  asm volatile("cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];"
               :: "r"(smem_u32(dst)), "l"(m), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile("cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
               :: "r"(smem_u32(dst)), "l"(m), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)) : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (canonical SW128 layout:
// 128-byte rows, 8-row groups 1024 bytes apart).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor: bf16 x bf16 -> f32, M x N, A/B major (0 = K, 1 = MN).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }"
               :: "r"(d), "l"(a), "l"(b), "r"(id), "r"(acc));
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }"
               :: "r"(d), "r"(a), "l"(b), "r"(id), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
         "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
         "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
         "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

struct TcParams {
  AttnArgs a;
  int mask_words;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
               const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mkb,
               const __grid_constant__ CUtensorMap mvb, const TcParams prm) {
  using C = Cfg<D>;
  const AttnArgs& a = prm.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::kTileBytes;
  uint8_t* sV = sK + kKStages * C::kTileBytes;
  Extra& x = *reinterpret_cast<Extra*>(sV + kVStages * C::kTileBytes);
  Bars& bar = x.bar;
  volatile int* abort_flag = &x.abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tq = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = (int64_t)b * a.H + h;
  const int i0 = 2 * tq;
  const int mw = prm.mask_words;

  // ---- set-up: barriers, TMEM, routing lists --------------------------------------------------
  if (tid == 0) {
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < kKStages; ++s) { mbar_init(&bar.k_full[s], 1); mbar_init(&bar.k_empty[s], 1); }
    for (int s = 0; s < kVStages; ++s) { mbar_init(&bar.v_full[s], 1); mbar_init(&bar.v_empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.s_full[s], 1); mbar_init(&bar.s_free[s], 4); mbar_init(&bar.p_full[s], 4);
      mbar_init(&bar.o_done[s], 1);
    }
    mbar_init(&bar.final_mma, 1);
    x.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" :: "r"(smem_u32(&x.tmem_base)), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  for (int w = tid; w < 2 * kMaxWords; w += kThreads) (&x.sel[0][0])[w] = 0u;
  const int n_tail = a.N - 64 * (a.nkb - 1);   // valid rows of the last key block
  for (int c = tid; c < 64; c += kThreads) x.tail_add[c] = c < n_tail ? 0.f : -INFINITY;
  __syncthreads();
  for (int hf = 0; hf < 2; ++hf) {
    const int i = i0 + hf;
    if (i >= a.nqb) continue;
    const int64_t row = bh * a.nqb + i;
    const int beg = a.row_ptr[row], end = a.row_ptr[row + 1];
    for (int e = beg + tid; e < end; e += kThreads) {
      const int j = a.col_idx[e];
      if (j >= 0 && j < a.nkb) atomicOr(&x.sel[hf][j >> 5], 1u << (j & 31));
      else raise_status(a.status, SOL_ERR_INVALID_ARG);
    }
  }
  __syncthreads();
  if (warp == 0) {
    // union list with per-half tags, ascending
    uint32_t ua = lane < mw ? x.sel[0][lane] : 0u, ub = lane < mw ? x.sel[1][lane] : 0u, u = ua | ub;
    int cnt = __popc(u), incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) { const int y = __shfl_up_sync(0xffffffffu, incl, o); if (lane >= o) incl += y; }
    int pos = incl - cnt;
    while (u) {
      const int bit = __ffs(u) - 1;
      u &= u - 1;
      x.list[pos++] = (32 * lane + bit) | (int)(((ua >> bit) & 1u) << 16) | (int)(((ub >> bit) & 1u) << 17);
    }
    if (lane == 31) x.n_union = incl;
    // centroid tiles holding at least one block unselected by a present half
    if (lane == 0) {
      x.present[0] = 1;
      x.present[1] = (i0 + 1 < a.nqb) ? 1 : 0;
      int n = 0;
      for (int ct = 0; ct * 128 < a.nkb; ++ct) {
        bool any = false;
        for (int w = 4 * ct; w < min(4 * ct + 4, mw); ++w) {
          const int valid = min(32, a.nkb - 32 * w);
          const uint32_t vm = valid >= 32 ? 0xffffffffu : ((1u << valid) - 1u);
          any |= ((~x.sel[0][w]) & vm) != 0u;
          if (x.present[1]) any |= ((~x.sel[1][w]) & vm) != 0u;
        }
        if (any) x.cent[n++] = ct;
      }
      x.n_cent = n;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < x.n_cent * 256; idx += kThreads) {
    const int slot = idx >> 8, hf = (idx >> 7) & 1, c = idx & 127;
    const int j = 128 * x.cent[slot] + c;
    const bool live = x.present[hf] && j < a.nkb && !((x.sel[hf][j >> 5] >> (j & 31)) & 1u);
    x.cent_add[slot][hf][c] = live ? a.cbias[bh * a.nkb + j] * kLog2e : -INFINITY;
  }
  __syncthreads();
  for (int idx = tid; idx < x.n_cent * 4; idx += kThreads) {
    const int slot = idx >> 2, hf = (idx >> 1) & 1, hh = idx & 1;
    int any = 0;
    for (int c = 0; c < 64; ++c) any |= x.cent_add[slot][hf][64 * hh + c] != -INFINITY;
    x.cent_live[slot][hf][hh] = any;
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = x.tmem_base;
  const int n_ex = (x.n_union + 1) >> 1;
  const int T = n_ex + x.n_cent;

  if (warp == 0 || warp == 6) {
    // ---------------------------------------------------------------- TMA producers
    // warp 0: Q and the K tiles (kKStages ring); warp 6: the V tiles
    // (kVStages ring).  Each runs ahead on its own ring.
    if (lane == 0) {
      const bool is_k = warp == 0;
      const int nst = is_k ? kKStages : kVStages;
      const CUtensorMap* m4 = is_k ? &mk : &mv;
      const CUtensorMap* m3 = is_k ? &mkb : &mvb;
      uint8_t* ring = is_k ? sK : sV;
      int nl = 0;   // tile loads issued
      bool ok = true;
      if (is_k) {
        mbar_expect_tx(&bar.q_full, C::kTileBytes);
        for (int hf = 0; hf < 2; ++hf)
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(sQ + c * C::kChunkBytes + hf * (C::kChunkBytes / 2), &mq, c * 64, h, 64 * (i0 + hf), b,
                        &bar.q_full);
      }
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % nst, n = t / nst;
        int j0 = 0, j1 = 0, ct = -1;
        if (t < n_ex) {
          j0 = x.list[2 * t] & 0xffff;
          j1 = (2 * t + 1 < x.n_union) ? (x.list[2 * t + 1] & 0xffff) : j0;
        } else {
          ct = x.cent[t - n_ex];
        }
        uint64_t* empty = is_k ? &bar.k_empty[s] : &bar.v_empty[s];
        uint64_t* full = is_k ? &bar.k_full[s] : &bar.v_full[s];
        if (!(ok = wait_bar(empty, (n & 1) ^ 1, abort_flag, a.status))) break;
        SOL_TRACE_AT(is_k ? 7 : 8, t);
        mbar_expect_tx(full, C::kTileBytes);
        ++nl;
        uint8_t* dst = ring + s * C::kTileBytes;
        for (int c = 0; c < C::kChunks; ++c) {
          if (ct < 0) {
            tma_load_4d(dst + c * C::kChunkBytes, m4, c * 64, h, 64 * j0, b, full);
            tma_load_4d(dst + c * C::kChunkBytes + C::kChunkBytes / 2, m4, c * 64, h, 64 * j1, b, full);
          } else {
            tma_load_3d(dst + c * C::kChunkBytes, m3, c * 64, 128 * ct, (int)bh, full);
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
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // Issue order QK(0), QK(1), QK(2), PV(0), QK(3), PV(1), QK(4), ...: the
    // tensor pipe runs in order and issuing blocks for about as long as the
    // MMAs take, so the QKs run ahead and S(u+1), S(u+2) are ready before the
    // softmax needs them.  QK(g) reuses S_(g%2) once the softmax has read
    // S(g-2) (it releases S right after loading it).
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t id_pv = idesc_bf16(128, D, 0, 1);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      const uint32_t o_tmem = tmem + 256;
      bool ok = wait_bar(&bar.q_full, 0, abort_flag, a.status);
      auto qk = [&](int g) -> bool {
        const int s = g % kKStages, n = g / kKStages, bb = g & 1;
        if (!wait_bar(&bar.k_full[s], n & 1, abort_flag, a.status)) return false;
        if (g >= 2 && !wait_bar(&bar.s_free[bb], ((g >> 1) - 1) & 1, abort_flag, a.status)) return false;
        fence_after();
        SOL_TRACE_AT(4, g);
        const uint32_t kb = k_addr + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
          mma_ss(tmem + bb * 128, sdesc(q_addr + off, 16, 1024), sdesc(kb + off, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar.s_full[bb]);
        mma_commit(&bar.k_empty[s]);
        return true;
      };
      auto pv = [&](int u) -> bool {
        const int s = u % kVStages, n = u / kVStages, bb = u & 1;
        if (!wait_bar(&bar.p_full[bb], (u >> 1) & 1, abort_flag, a.status)) return false;
        SOL_TRACE_AT(5, u);
        if (!wait_bar(&bar.v_full[s], n & 1, abort_flag, a.status)) return false;
        fence_after();
        const uint32_t vb = v_addr + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(o_tmem, tmem + 384 + 64 * bb + kk * 8, sdesc(vb + kk * 2048, C::kChunkBytes, 1024), id_pv,
                 (u > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar.v_empty[s]);
        mma_commit(&bar.o_done[bb]);
        return true;
      };
      for (int g = 0; g < 3 && g < T && ok; ++g) ok = qk(g);
      for (int u = 0; u < T && ok; ++u) {
        ok = pv(u);
        if (ok && u + 3 < T) ok = qk(u + 3);
      }
      // drain: all issued MMAs complete before TMEM is released
      mma_commit(&bar.final_mma);
      drain_bar(&bar.final_mma, 0, a.status);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ---------------------------------------------------------------- softmax warpgroup
    // One pass per S tile: the needed columns are read once (S is then
    // released to the next QK), masked, maxed, exponentiated and stored as bf16
    // P into its own TMEM buffer P_(u%2), once PV(u-2), the last reader of
    // that buffer, is complete.  PV completions are waited for only there, for
    // a rescale of O (PV(u-1)) and before the epilogue (PV(T-1)).  PV(v)
    // completes o_done[v%2]; the next completion of that barrier needs P(v+2),
    // which this warpgroup has not produced yet, so each parity wait is exact.
    const int sub = warp & 3;                 // TMEM sub-partition = rows 32*sub .. 32*sub+31
    const int r = 32 * sub + lane;            // row of the tile
    const int hf = r >> 6;                    // query block half (warp-uniform)
    const bool present = x.present[hf] != 0;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * sub) << 16);
    const uint32_t o_addr = lane_addr + 256;
    const float sl2 = a.scale * kLog2e;
    const bool tracer = warp == 2 && lane == 0;
    float m_run = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int bb = t & 1;
      ok = __all_sync(0xffffffffu, wait_bar(&bar.s_full[bb], (t >> 1) & 1, abort_flag, a.status));
      if (!ok) break;
      fence_after();
      if (tracer) SOL_TRACE_AT(0, t);
      // which 64-column halves of this S tile the row uses, and their additive offsets
      bool need0, need1;
      const float *add0, *add1;
      if (t < n_ex) {
        const int e0 = x.list[2 * t];
        const int e1 = (2 * t + 1 < x.n_union) ? x.list[2 * t + 1] : -1;
        need0 = present && ((e0 >> (16 + hf)) & 1);
        need1 = present && e1 >= 0 && ((e1 >> (16 + hf)) & 1);
        add0 = ((e0 & 0xffff) == a.nkb - 1) ? x.tail_add : nullptr;
        add1 = (e1 >= 0 && (e1 & 0xffff) == a.nkb - 1) ? x.tail_add : nullptr;
      } else {
        const int slot = t - n_ex;
        need0 = x.cent_live[slot][hf][0] != 0;
        need1 = x.cent_live[slot][hf][1] != 0;
        add0 = x.cent_add[slot][hf];
        add1 = x.cent_add[slot][hf] + 64;
      }
      const uint32_t s_addr = lane_addr + bb * 128;
      float sv[128];
      if (need0) { tmem_ld32(s_addr, sv); tmem_ld32(s_addr + 32, sv + 32); }
      if (need1) { tmem_ld32(s_addr + 64, sv + 64); tmem_ld32(s_addr + 96, sv + 96); }
      tmem_wait_ld();
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.s_free[bb]);
      // logits in log2 units (masked / offset) and the tile's row max
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (!(hh ? need1 : need0)) continue;
        const float* ad = hh ? add1 : add0;
        if (ad) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            sv[64 * hh + c] = fmaf(sv[64 * hh + c], sl2, ad[c]);
            m4[c & 3] = fmaxf(m4[c & 3], sv[64 * hh + c]);
          }
        } else {
          float r4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 64; ++c) r4[c & 3] = fmaxf(r4[c & 3], sv[64 * hh + c]);
#pragma unroll
          for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], r4[q] * sl2);
        }
      }
      const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      if (tracer) SOL_TRACE_AT(1, t);
      float alpha = 1.f;
      bool resc = false;
      if (mt > m_run + kRescale || (m_run == -INFINITY && mt != -INFINITY)) {
        alpha = ex2(m_run - mt);            // 0 when m_run = -inf
        resc = l > 0.f;
        l *= alpha;
        m_run = mt;
      }
      const float base = (m_run == -INFINITY) ? 0.f : m_run;
      if (t >= 2) {   // P_bb's previous reader, PV(t-2)
        ok = __all_sync(0xffffffffu, wait_bar(&bar.o_done[bb], ((t - 2) >> 1) & 1, abort_flag, a.status));
        if (!ok) break;
        fence_after();
      }
      // p = 2^(x - base) as bf16 pairs into P_bb
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t pk[32];
        if (hh ? need1 : need0) {
          const bool scaled = (hh ? add1 : add0) != nullptr;   // logits already in log2 units
          const float mul = scaled ? 1.f : sl2;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float p0 = ex2(fmaf(sv[64 * hh + 2 * c], mul, -base));
            const float p1 = ex2(fmaf(sv[64 * hh + 2 * c + 1], mul, -base));
            l4[c & 3] += p0 + p1;
            pk[c] = pack_bf16(p0, p1);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = 0u;
        }
        tmem_st32(lane_addr + 384 + 64 * bb + 32 * hh, pk);
      }
      l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      if (tracer) SOL_TRACE_AT(2, t);
      // O is rescaled only once PV(t-1), the last MMA to accumulate into it, is complete
      if (t >= 1 && __any_sync(0xffffffffu, resc)) {
        ok = __all_sync(0xffffffffu, wait_bar(&bar.o_done[(t - 1) & 1], ((t - 1) >> 1) & 1, abort_flag, a.status));
        if (!ok) break;
        fence_after();
        const float f = resc ? alpha : 1.f;
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
      tmem_wait_st();
      fence_before();
      __syncwarp();
      if (tracer) SOL_TRACE_AT(3, t);
      if (lane == 0) mbar_arrive(&bar.p_full[bb]);
    }
    // epilogue: O / l -> bf16, once the last PV is complete
    if (ok && T > 0)
      ok = __all_sync(0xffffffffu, wait_bar(&bar.o_done[(T - 1) & 1], ((T - 1) >> 1) & 1, abort_flag, a.status));
    if (ok) {
      fence_after();
      const int grow = 64 * (i0 + hf) + (r & 63);
      const bool store = present && grow < a.N;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = a.o + (int64_t)b * a.ob + (int64_t)h * a.oh + (int64_t)grow * a.on;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float ov[32];
        tmem_ld32(o_addr + 32 * c, ov);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 u4 = make_uint4(pack_bf16(ov[e] * inv, ov[e + 1] * inv), pack_bf16(ov[e + 2] * inv, ov[e + 3] * inv),
                                  pack_bf16(ov[e + 4] * inv, ov[e + 5] * inv), pack_bf16(ov[e + 6] * inv, ov[e + 7] * inv));
            *reinterpret_cast<uint4*>(orow + 32 * c + e) = u4;
          }
        }
      }
      if (store && a.lse) a.lse[bh * a.N + grow] = (m_run + log2f(l)) * kLn2;
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(512));
  }
}

// ---- host side: tensor maps and launch ------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
              const cuuint32_t* box) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_tc(const AttnArgs& a, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mkb, mvb;
  const cuuint64_t bstride = (cuuint64_t)(a.B > 1 ? a.sb : (int64_t)a.N * a.sn) * 2;
  const cuuint64_t dims4[4] = {(cuuint64_t)D, (cuuint64_t)a.H, (cuuint64_t)a.N, (cuuint64_t)a.B};
  const cuuint64_t str4[3] = {(cuuint64_t)a.sh * 2, (cuuint64_t)a.sn * 2, bstride};
  const cuuint32_t box4[4] = {64, 1, 64, 1};
  const cuuint64_t dims3[3] = {(cuuint64_t)D, (cuuint64_t)a.nkb, (cuuint64_t)a.B * a.H};
  const cuuint64_t str3[2] = {(cuuint64_t)D * 2, (cuuint64_t)a.nkb * D * 2};
  const cuuint32_t box3[3] = {64, 128, 1};
  if (!make_map(&mq, a.q, 4, dims4, str4, box4) || !make_map(&mk, a.k, 4, dims4, str4, box4) ||
      !make_map(&mv, a.v, 4, dims4, str4, box4) || !make_map(&mkb, a.kbar16, 3, dims3, str3, box3) ||
      !make_map(&mvb, a.vbar16, 3, dims3, str3, box3))
    return cudaErrorInvalidValue;
  TcParams prm{a, (a.nkb + 31) / 32};
  const size_t smem = 1024 + Cfg<D>::kSmemTiles + sizeof(Extra);
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.nqb + 1) / 2, a.H, a.B);
  attn_tc_kernel<D><<<grid, kThreads, smem, st>>>(mq, mk, mv, mkb, mvb, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn(const AttnArgs& a, int D, cudaStream_t st) {
  return D == 128 ? launch_tc<128>(a, st) : launch_tc<64>(a, st);
}

}  // namespace sol

#ifdef SOL_TRACE
// Copies the phase trace (16 slots x 256 steps of clock64 stamps) to host memory.
extern "C" int sol_debug_trace(long long* host, int n) {
  const int total = 16 * sol::kTraceSteps;
  return (int)cudaMemcpyFromSymbol(host, sol::g_trace, sizeof(long long) * (n < total ? n : total));
}
#endif
