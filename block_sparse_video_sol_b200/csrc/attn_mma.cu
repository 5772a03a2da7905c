// sol_attn_fwd, first correct path: exact + centroid attention on mma.sync.
//
// Star7 README "MiniMax H3 Activation Chunk & Attention Acceleration",
// section 工作原理 > Sol: selected K/V blocks are attended exactly; each
// unselected block contributes through its K/V centroid, and both kinds of
// term are merged in the same FP32 online softmax.
//
// One CTA per (query block i, head h, batch b); 4 warps, 16 query rows each.
// The tile sequence of a CTA is its CSR list of exact key blocks (64 keys
// each, rows >= N masked) followed by the chunks of 64 centroids that hold at
// least one unselected block (selected ones masked, logit offset
// log n_j (+ bias_j) added).  K/V tiles are double-buffered with cp.async.
#include <math.h>

#include "common.cuh"

namespace sol {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(smem_addr(dst)), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_addr(p)));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Swizzled element offset of (row, 16-byte chunk) in a [64][D] bf16 tile.
template <int D> __device__ __forceinline__ int swz(int r, int ch) { return r * D + ((ch ^ (r & 7)) << 3); }

}  // namespace

template <int D>
__global__ void __launch_bounds__(128) attn_mma_kernel(const AttnArgs a) {
  constexpr int CH = D / 8;
  constexpr int TILE = 64 * D;
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sK = sQ + TILE;          // [2][64][D]
  __nv_bfloat16* sV = sK + 2 * TILE;      // [2][64][D]
  uint32_t* sSel = reinterpret_cast<uint32_t*>(sV + 2 * TILE);   // [kMaxKeyBlocks/32]
  int* sList = reinterpret_cast<int*>(sSel + kMaxKeyBlocks / 32); // exact blocks, then centroid chunks
  __shared__ int sNumChunks;

  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int64_t bh = (int64_t)b * a.H + h;
  const int64_t row = bh * a.nqb + i;
  const int beg = a.row_ptr[row], n_exact = a.row_ptr[row + 1] - beg;
  const int mask_words = (a.nkb + 31) / 32, n_chunks_all = (a.nkb + 63) / 64;

  for (int w = tid; w < mask_words; w += 128) sSel[w] = 0u;
  __syncthreads();
  for (int e = tid; e < n_exact; e += 128) {
    const int j = a.col_idx[beg + e];
    if (j >= 0 && j < a.nkb) { atomicOr(&sSel[j >> 5], 1u << (j & 31)); sList[e] = j; }
    else { raise_status(a.status, SOL_ERR_INVALID_ARG); sList[e] = -1; }
  }
  __syncthreads();
  if (tid == 0) {
    int n = 0;
    for (int c = 0; c < n_chunks_all; ++c) {
      bool any = false;
      for (int w = 2 * c; w < min(2 * c + 2, mask_words); ++w) {
        const int valid = min(32, a.nkb - 32 * w);
        const uint32_t vm = valid >= 32 ? 0xffffffffu : ((1u << valid) - 1u);
        any |= ((~sSel[w]) & vm) != 0u;
      }
      if (any) sList[n_exact + n++] = c;
    }
    sNumChunks = n;
  }
  __syncthreads();
  const int n_tiles = n_exact + sNumChunks;

  const __nv_bfloat16* qbase = a.q + (int64_t)b * a.sb + (int64_t)h * a.sh;
  const __nv_bfloat16* kbase = a.k + (int64_t)b * a.sb + (int64_t)h * a.sh;
  const __nv_bfloat16* vbase = a.v + (int64_t)b * a.sb + (int64_t)h * a.sh;
  {
    const int q0 = i * 64, qv = min(64, a.N - q0);
    for (int idx = tid; idx < 64 * CH; idx += 128) {
      const int r = idx / CH, ch = idx % CH;
      const int rr = r < qv ? r : 0;
      cp_async16(sQ + swz<D>(r, ch), qbase + (int64_t)(q0 + rr) * a.sn + ch * 8, r < qv ? 16 : 0);
    }
    cp_async_commit();
  }
  auto load_tile = [&](int u, int stage) {
    const __nv_bfloat16 *ks, *vs;
    int64_t stride;
    int valid;
    if (u < n_exact) {
      const int j = max(sList[u], 0);
      ks = kbase + (int64_t)j * 64 * a.sn;
      vs = vbase + (int64_t)j * 64 * a.sn;
      stride = a.sn;
      valid = min(64, a.N - j * 64);
    } else {
      const int c = sList[u];
      ks = a.kbar16 + (bh * a.nkb + (int64_t)c * 64) * D;
      vs = a.vbar16 + (bh * a.nkb + (int64_t)c * 64) * D;
      stride = D;
      valid = min(64, a.nkb - c * 64);
    }
    __nv_bfloat16* dk = sK + stage * TILE;
    __nv_bfloat16* dv = sV + stage * TILE;
    for (int idx = tid; idx < 64 * CH; idx += 128) {
      const int r = idx / CH, ch = idx % CH;
      const int rr = r < valid ? r : 0;
      cp_async16(dk + swz<D>(r, ch), ks + rr * stride + ch * 8, r < valid ? 16 : 0);
      cp_async16(dv + swz<D>(r, ch), vs + rr * stride + ch * 8, r < valid ? 16 : 0);
    }
    cp_async_commit();
  };
  if (n_tiles > 0) load_tile(0, 0); else cp_async_commit();

  uint32_t qf[D / 16][4];
  float o[D / 8][4];
#pragma unroll
  for (int dt = 0; dt < D / 8; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // rows g and g+8 of this warp
  const float sl2 = a.scale * kLog2e;

  for (int u = 0; u < n_tiles; ++u) {
    if (u + 1 < n_tiles) load_tile(u + 1, (u + 1) & 1); else cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (u == 0) {
#pragma unroll
      for (int kd = 0; kd < D / 16; ++kd)
        ldsm_x4(qf[kd][0], qf[kd][1], qf[kd][2], qf[kd][3], sQ + swz<D>(16 * warp + (lane & 15), 2 * kd + (lane >> 4)));
    }
    const bool exact = u < n_exact;
    if (exact && sList[u] < 0) { __syncthreads(); continue; }
    const __nv_bfloat16* tk = sK + (u & 1) * TILE;
    const __nv_bfloat16* tv = sV + (u & 1) * TILE;

    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kd = 0; kd < D / 16; ++kd) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int key = 16 * np + (lane & 7) + ((lane >> 4) << 3);
        ldsm_x4(b0, b1, b2, b3, tk + swz<D>(key, 2 * kd + ((lane >> 3) & 1)));
        mma16816(s[2 * np], qf[kd], b0, b1);
        mma16816(s[2 * np + 1], qf[kd], b2, b3);
      }
    }
    // logits in log2 units, with the per-column offset / mask of this tile
    float add[8][2];
    if (exact) {
      const int key0 = sList[u] * 64;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) add[nt][e] = (key0 + 8 * nt + 2 * t4 + e < a.N) ? 0.f : -INFINITY;
    } else {
      const int c0 = sList[u] * 64;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int jc = c0 + 8 * nt + 2 * t4 + e;
          const bool live = jc < a.nkb && !((sSel[jc >> 5] >> (jc & 31)) & 1u);
          add[nt][e] = live ? a.cbias[bh * a.nkb + jc] * kLog2e : -INFINITY;
        }
    }
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = fmaf(s[nt][0], sl2, add[nt][0]);
      s[nt][1] = fmaf(s[nt][1], sl2, add[nt][1]);
      s[nt][2] = fmaf(s[nt][2], sl2, add[nt][0]);
      s[nt][3] = fmaf(s[nt][3], sl2, add[nt][1]);
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float base0 = (mx0 == -INFINITY) ? 0.f : mx0;
    const float base1 = (mx1 == -INFINITY) ? 0.f : mx1;
    const float al0 = exp2f(m0 - base0), al1 = exp2f(m1 - base1);
    m0 = mx0; m1 = mx1;
    l0 *= al0; l1 *= al1;
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) { o[dt][0] *= al0; o[dt][1] *= al0; o[dt][2] *= al1; o[dt][3] *= al1; }
    uint32_t pf[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = exp2f(s[nt][0] - base0), p1 = exp2f(s[nt][1] - base0);
      const float p2 = exp2f(s[nt][2] - base1), p3 = exp2f(s[nt][3] - base1);
      l0 += p0 + p1; l1 += p2 + p3;
      pf[nt >> 1][(nt & 1) * 2 + 0] = pack2(p0, p1);
      pf[nt >> 1][(nt & 1) * 2 + 1] = pack2(p2, p3);
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t b0, b1, b2, b3;
        const int key = 16 * ks + (lane & 7) + (((lane >> 3) & 1) << 3);
        ldsm_x4_t(b0, b1, b2, b3, tv + swz<D>(key, 2 * dp + (lane >> 4)));
        mma16816(o[2 * dp], pf[ks], b0, b1);
        mma16816(o[2 * dp + 1], pf[ks], b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
  const int r0 = i * 64 + 16 * warp + g, r1 = r0 + 8;
  __nv_bfloat16* obase = a.o + (int64_t)b * a.ob + (int64_t)h * a.oh;
#pragma unroll
  for (int dt = 0; dt < D / 8; ++dt) {
    const int d = 8 * dt + 2 * t4;
    if (r0 < a.N) *reinterpret_cast<uint32_t*>(obase + (int64_t)r0 * a.on + d) = pack2(o[dt][0] * inv0, o[dt][1] * inv0);
    if (r1 < a.N) *reinterpret_cast<uint32_t*>(obase + (int64_t)r1 * a.on + d) = pack2(o[dt][2] * inv1, o[dt][3] * inv1);
  }
  if (a.lse && t4 == 0) {
    if (r0 < a.N) a.lse[bh * a.N + r0] = (m0 + log2f(l0)) * kLn2;
    if (r1 < a.N) a.lse[bh * a.N + r1] = (m1 + log2f(l1)) * kLn2;
  }
}

cudaError_t launch_attn(const AttnArgs& a, int D, cudaStream_t st) {
  dim3 grid(a.nqb, a.H, a.B);
  cudaError_t e;
  if (D == 128) {
    const size_t smem = 5 * 64 * 128 * 2 + kMaxKeyBlocks / 8 + (kMaxKeyBlocks + kMaxKeyBlocks / 64) * 4;
    e = cudaFuncSetAttribute(attn_mma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attn_mma_kernel<128><<<grid, 128, smem, st>>>(a);
  } else {
    const size_t smem = 5 * 64 * 64 * 2 + kMaxKeyBlocks / 8 + (kMaxKeyBlocks + kMaxKeyBlocks / 64) * 4;
    e = cudaFuncSetAttribute(attn_mma_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attn_mma_kernel<64><<<grid, 128, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sol
