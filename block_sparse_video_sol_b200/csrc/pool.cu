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

// Anchor-weighted key/value summaries (Spark-H3 news page, Spark-Reweight
// bullet: the compressed branch's mean-pooled summaries become weighted ones,
// scored against one anchor per head).  Within key block j the weights are the
// anchor's softmax over the block's rows, w_t = exp(s a.k_t) / sum_u exp(s a.k_u);
// the centroid key and value the attention sees are ktil_j = sum_t w_t k_t and
// vtil_j = sum_t w_t v_t (bf16), and the centroid-logit offset is
// log n_j + bias_j = logsumexp_t(s a.k_t) - s a.ktil_j, so a query equal to the
// anchor receives the block's exact contribution.  The fp32 mean of K is still
// written: routing scores the mean-pooled centroids.
//
// One pass reads each K and V element once (the same HBM bytes as the mean
// pooling of K and V): a thread owns 8 dims of one head of both tensors, keeps
// 8 K rows and 8 V rows (16 x 16 B) in flight, and folds each group of 8 rows
// into an online softmax (one rescale per group).  The dot a.k_t is reduced
// over the head's TPH lanes with an xor butterfly, which leaves the bitwise
// same value in every lane, so the online state is uniform over a head.
template <int D, int HPB>
__global__ void __launch_bounds__(HPB * (D / 8)) pool_kv_reweight_kernel(const PoolArgs a) {
  constexpr int TPH = D / 8;  // threads per head
  const int j = blockIdx.x;
  const int h = blockIdx.y * HPB + threadIdx.x / TPH;
  const int c = threadIdx.x % TPH;
  const int b = blockIdx.z;
  const bool active = h < a.H;
  const int r0 = j * kBlock, r1 = min(a.N, r0 + kBlock), n = r1 - r0;
  const int64_t off = (int64_t)b * a.sb + (int64_t)h * a.sh + c * 8;
  const __nv_bfloat16* kb = a.src[1] + off;
  const __nv_bfloat16* vb = a.src[2] + off;

  float an[8], mean[8], wk[8], wv[8], m = -INFINITY, l = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    an[i] = active ? a.anchor[((int64_t)b * a.H + h) * D + c * 8 + i] : 0.f;
    mean[i] = wk[i] = wv[i] = 0.f;
  }

  for (int r = r0; r < r1; r += 8) {
    uint4 uk[8], uv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uk[k] = uv[k] = make_uint4(0, 0, 0, 0);
      if (active && r + k < r1) {
        uk[k] = __ldg(reinterpret_cast<const uint4*>(kb + (int64_t)(r + k) * a.sn));
        uv[k] = __ldg(reinterpret_cast<const uint4*>(vb + (int64_t)(r + k) * a.sn));
      }
    }
    float x[8], gmax = m;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float f[8], dot = 0.f;
      bf16x8_to_f32(uk[k], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        mean[i] += f[i];
        dot = fmaf(an[i], f[i], dot);
      }
#pragma unroll
      for (int o = TPH / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      x[k] = (r + k < r1) ? a.scale * dot : -INFINITY;  // uniform over the CTA
      gmax = fmaxf(gmax, x[k]);
    }
    // gmax is finite: row r is valid.  expf(-inf) = 0 covers the first group.
    const float corr = expf(m - gmax);
    m = gmax;
    l *= corr;
#pragma unroll
    for (int i = 0; i < 8; ++i) { wk[i] *= corr; wv[i] *= corr; }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float e = expf(x[k] - m);
      float fk[8], fv[8];
      bf16x8_to_f32(uk[k], fk);
      bf16x8_to_f32(uv[k], fv);
      l += e;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        wk[i] = fmaf(e, fk[i], wk[i]);
        wv[i] = fmaf(e, fv[i], wv[i]);
      }
    }
  }
  if (n <= 0) return;  // uniform over the CTA
  const float inv_n = 1.f / (float)n, inv_l = 1.f / l;
  float pooled = 0.f;  // s * a.ktil, reduced over the head's lanes (every lane takes part)
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mean[i] *= inv_n;
    wk[i] *= inv_l;
    wv[i] *= inv_l;
    pooled = fmaf(an[i], wk[i], pooled);
  }
#pragma unroll
  for (int o = TPH / 2; o > 0; o >>= 1) pooled += __shfl_xor_sync(0xffffffffu, pooled, o);
  if (!active) return;
  const int64_t row = ((int64_t)b * a.H + h) * a.nb + j;
  float* dst = a.kbar + row * D + c * 8;
  reinterpret_cast<float4*>(dst)[0] = make_float4(mean[0], mean[1], mean[2], mean[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(mean[4], mean[5], mean[6], mean[7]);
  reinterpret_cast<uint4*>(a.kbar16 + row * D + c * 8)[0] =
      make_uint4(pack_bf16x2(wk[0], wk[1]), pack_bf16x2(wk[2], wk[3]), pack_bf16x2(wk[4], wk[5]),
                 pack_bf16x2(wk[6], wk[7]));
  reinterpret_cast<uint4*>(a.vbar16 + row * D + c * 8)[0] =
      make_uint4(pack_bf16x2(wv[0], wv[1]), pack_bf16x2(wv[2], wv[3]), pack_bf16x2(wv[4], wv[5]),
                 pack_bf16x2(wv[6], wv[7]));
  if (c == 0) a.cbias[row] = m + logf(l) - a.scale * pooled;
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

cudaError_t launch_pool_kv_reweight(const PoolArgs& a, int D, cudaStream_t st) {
  if (D == 128) {
    constexpr int HPB = 8;
    dim3 grid(a.nb, (a.H + HPB - 1) / HPB, a.B);
    pool_kv_reweight_kernel<128, HPB><<<grid, HPB * 16, 0, st>>>(a);
  } else {
    constexpr int HPB = 16;
    dim3 grid(a.nb, (a.H + HPB - 1) / HPB, a.B);
    pool_kv_reweight_kernel<64, HPB><<<grid, HPB * 8, 0, st>>>(a);
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
