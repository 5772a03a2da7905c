// sol_pool kernels: block centroids of Q, K, V and the optional log-mass bias.
//
// Block centroids ("K/V centroids") follow the Star7 README "MiniMax H3
// Activation Chunk & Attention Acceleration", section 工作原理 > Sol; the
// log-mass bias follows the Spark-H3 news page (comfyui-wiki), Spark-Reweight
// bullet: mean pooling yields exp(E[x]) rather than E[exp(x)], a per-block
// bias restores the missing mass, scored against one anchor per head (the
// mean video query).
//
// The pass is HBM-bound: every input element is read exactly once.  A CTA
// owns one 64-row block of HPB heads; each thread owns one 16-byte chunk
// (8 bf16) of one head and streams the block's rows with 8 independent
// 16-byte loads in flight, accumulating in fp32.
#include <math.h>

#include "common.cuh"

namespace sol {

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D, int HPB>
__global__ void __launch_bounds__(HPB * (D / 8)) pool_kernel(const PoolArgs a) {
  constexpr int TPH = D / 8;  // threads per head
  const int j = blockIdx.x;
  const int h = blockIdx.y * HPB + threadIdx.x / TPH;
  const int c = threadIdx.x % TPH;
  const int nt = __popc(a.tensor_mask);
  const int b = blockIdx.z / nt;
  int slot = blockIdx.z % nt, t = 0;
  for (int m = a.tensor_mask; ; m &= m - 1) {  // t = index of the slot-th set bit
    if (slot-- == 0) { t = __ffs(m) - 1; break; }
  }
  const bool active = h < a.H;
  const int r0 = j * kBlock, r1 = min(a.N, r0 + kBlock), n = r1 - r0;
  const __nv_bfloat16* src = t == 0 ? a.src[0] : (t == 1 ? a.src[1] : a.src[2]);
  const __nv_bfloat16* base = src + (int64_t)b * a.sb + (int64_t)h * a.sh + c * 8;
  const bool bias = (t == 1) && a.with_bias;

  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  float an[8], m = -INFINITY, l = 0.f;
  if (bias) {
#pragma unroll
    for (int i = 0; i < 8; ++i) an[i] = active ? a.anchor[((int64_t)b * a.H + h) * D + c * 8 + i] : 0.f;
  }

  for (int r = r0; r < r1; r += 8) {
    uint4 u[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      u[k] = make_uint4(0, 0, 0, 0);
      if (active && r + k < r1) u[k] = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)(r + k) * a.sn));
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float f[8];
      bf16x8_to_f32(u[k], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += f[i];
      if (bias) {
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) dot = fmaf(an[i], f[i], dot);
#pragma unroll
        for (int off = TPH / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        if (r + k < r1) {  // uniform over the CTA
          const float x = a.scale * dot;
          if (x > m) { l = l * expf(m - x) + 1.f; m = x; }
          else l += expf(x - m);
        }
      }
    }
  }
  if (n <= 0) return;  // uniform over the CTA
  const float inv = 1.f / (float)n;
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] *= inv;
  float pooled = 0.f;  // s * a.kbar, reduced over the head's lanes (every lane takes part)
  if (bias) {
#pragma unroll
    for (int i = 0; i < 8; ++i) pooled = fmaf(an[i], acc[i], pooled);
#pragma unroll
    for (int off = TPH / 2; off > 0; off >>= 1) pooled += __shfl_xor_sync(0xffffffffu, pooled, off);
    pooled *= a.scale;
  }
  if (!active) return;
  const int64_t row = ((int64_t)b * a.H + h) * a.nb + j;
  if (t == 0 || t == 1) {
    float* dst = (t == 0 ? a.qbar : a.kbar) + row * D + c * 8;
    reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  if (t == 1 || t == 2) {
    uint4 pk = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                          pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    reinterpret_cast<uint4*>((t == 1 ? a.kbar16 : a.vbar16) + row * D + c * 8)[0] = pk;
  }
  if (t == 1) {
    // log n + (log mean_t exp(s a.k_t) - s a.kbar) = logsumexp_t(s a.k_t) - s a.kbar
    const float off = bias ? (m + logf(l) - pooled) : logf((float)n);
    if (c == 0) a.cbias[row] = off;
  }
}

// Anchor a = mean of the query rows >= prefix (all rows when prefix >= N),
// from the pooled Q block means plus the rows of the block the prefix ends in.
template <int D>
__global__ void __launch_bounds__(D) anchor_kernel(const __nv_bfloat16* q, int64_t sb, int64_t sn, int64_t sh,
                                                   const float* qbar, int N, int H, int nqb, int prefix,
                                                   float* anchor) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int P = prefix < N ? prefix : 0;
  const int first = (P + kBlock - 1) / kBlock;
  const float* qb = qbar + ((int64_t)b * H + h) * nqb * D + d;
  float acc = 0.f;
  for (int i = first; i < nqb; ++i) acc += qb[(int64_t)i * D] * (float)(min(N, (i + 1) * kBlock) - i * kBlock);
  const __nv_bfloat16* qr = q + (int64_t)b * sb + (int64_t)h * sh + d;
  for (int r = P; r < min(N, first * kBlock); ++r) acc += __bfloat162float(qr[(int64_t)r * sn]);
  anchor[((int64_t)b * H + h) * D + d] = acc / (float)(N - P);
}

cudaError_t launch_pool(const PoolArgs& a, int D, cudaStream_t st) {
  const int nt = __builtin_popcount(a.tensor_mask);
  if (D == 128) {
    constexpr int HPB = 8;
    dim3 grid(a.nb, (a.H + HPB - 1) / HPB, a.B * nt);
    pool_kernel<128, HPB><<<grid, HPB * 16, 0, st>>>(a);
  } else {
    constexpr int HPB = 16;
    dim3 grid(a.nb, (a.H + HPB - 1) / HPB, a.B * nt);
    pool_kernel<64, HPB><<<grid, HPB * 8, 0, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_anchor(const __nv_bfloat16* q, int64_t sb, int64_t sn, int64_t sh, const float* qbar,
                          int B, int N, int H, int D, int nqb, int prefix, float* anchor, cudaStream_t st) {
  dim3 grid(H, B);
  if (D == 128) anchor_kernel<128><<<grid, 128, 0, st>>>(q, sb, sn, sh, qbar, N, H, nqb, prefix, anchor);
  else anchor_kernel<64><<<grid, 64, 0, st>>>(q, sb, sn, sh, qbar, N, H, nqb, prefix, anchor);
  return cudaGetLastError();
}

}  // namespace sol
