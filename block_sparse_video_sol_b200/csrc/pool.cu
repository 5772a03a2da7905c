// sol_pool kernels: block centroids of Q, K, V, the anchor, the optional
// log-mass bias and the optional anchor-weighted key/value summaries.
//
// Block centroids ("K/V centroids") follow the Star7 README "MiniMax H3
// Activation Chunk & Attention Acceleration", section 工作原理 > Sol; the
// log-mass bias follows the Spark-H3 news page (comfyui-wiki), Spark-Reweight
// bullet: mean pooling yields exp(E[x]) rather than E[exp(x)], a per-block
// bias restores the missing mass, scored against one anchor per head (the
// mean video query).
//
// The mean pass is HBM-bound: every input element is read exactly once.  A CTA
// owns one 64-row block of HPB heads; each thread owns one 16-byte chunk
// (8 bf16) of one head and streams the block's rows with 8 independent
// 16-byte loads in flight, accumulating in fp32.
#include <math.h>

#include "common.cuh"
#include "ptx.cuh"   // packed f32x2 arithmetic

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
// One pass reads each K and V element once.  A CTA owns one key block of
// kHeads heads; a thread owns 8 dims (one 16-byte chunk) of one head and
// streams the block's rows in groups of 4 (8 loads in flight), folding each
// group into an online softmax:
//   - partial dots of the 4 rows with the anchor, reduced over the head's
//     chunk lanes by a transposing butterfly that leaves each lane one row's
//     full dot (5 shuffles for 4 rows instead of 16);
//   - the group's max (2 shuffles), one rescale of the running sums per
//     group, and the 4 rows' weights gathered back to every lane (4 shuffles);
//   - key sum, weighted key and weighted value in packed f32x2 arithmetic.
// No shared memory and no barrier: warps are independent and hide each
// other's load latency (about 120 registers, four CTAs per SM).  Measured against
// this form on B200: a TMA-staged one-tile CTA, and persistent TMA-ring CTAs
// (with and without a producer warp) whose barrier-separated phases left
// each tile's critical path too long; both were slower.
template <int D>
struct RwCfg {
  static constexpr int kChunks = D / 8;            // lanes per head
  static constexpr int kThreads = 128;
  static constexpr int kHeads = kThreads / kChunks;   // heads per CTA: 8 (D = 128) or 16 (D = 64)
};

template <int D>
__global__ void __launch_bounds__(128, 4) pool_kv_reweight_kernel(const PoolArgs a) {
  using C = RwCfg<D>;
  constexpr int CH = C::kChunks, B1 = CH / 2, B2 = CH / 4;
  const int lane = threadIdx.x % 32;
  const int j = blockIdx.x;
  const int h = blockIdx.y * C::kHeads + threadIdx.x / CH;
  const int c = threadIdx.x % CH;
  const int b = blockIdx.z;
  const bool active = h < a.H;
  const int r0 = j * kBlock, r1 = min(a.N, r0 + kBlock), n = r1 - r0;
  const int64_t off = (int64_t)b * a.sb + (int64_t)h * a.sh + c * 8;
  const __nv_bfloat16* kb = a.src[1] + off;
  const __nv_bfloat16* vb = a.src[2] + off;

  uint64_t an2[4];   // this chunk of the anchor, as packed pairs
  {
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
    if (active) {
      a0 = *reinterpret_cast<const float4*>(a.anchor + ((int64_t)b * a.H + h) * D + c * 8);
      a1 = *reinterpret_cast<const float4*>(a.anchor + ((int64_t)b * a.H + h) * D + c * 8 + 4);
    }
    an2[0] = f2pack(a0.x, a0.y);
    an2[1] = f2pack(a0.z, a0.w);
    an2[2] = f2pack(a1.x, a1.y);
    an2[3] = f2pack(a1.z, a1.w);
  }
  // After the butterfly this lane holds the full dot of row `own` of a group;
  // the lanes holding rows 0..3 differ from it only in bits B1 and B2.
  const bool b1 = lane & B1, b2 = lane & B2;
  const int own = (b1 ? 2 : 0) + (b2 ? 1 : 0);
  const int base_lane = lane & ~(B1 | B2);

  auto load = [&](int r, uint4* kr, uint4* vr) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      kr[i] = vr[i] = make_uint4(0, 0, 0, 0);
      if (active && r + i < r1) {
        kr[i] = __ldg(reinterpret_cast<const uint4*>(kb + (int64_t)(r + i) * a.sn));
        vr[i] = __ldg(reinterpret_cast<const uint4*>(vb + (int64_t)(r + i) * a.sn));
      }
    }
  };
  auto pair = [](uint32_t w) { return f2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)); };
  auto word = [](const uint4& u, int e) { return e == 0 ? u.x : e == 1 ? u.y : e == 2 ? u.z : u.w; };

  uint64_t sk[4] = {0, 0, 0, 0}, wk[4] = {0, 0, 0, 0}, wv[4] = {0, 0, 0, 0};   // packed (0.f, 0.f)
  float m = -INFINITY, l = 0.f;
  // The next group's loads are issued at the end of each iteration (measured
  // on B200: the same loop with the loads at its top ran 35% slower).
  uint4 kr[4], vr[4];
  load(r0, kr, vr);
  for (int r = r0; r < r1; r += 4) {   // uniform over the CTA
    uint64_t k2[4][4];
    float p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint64_t acc = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        k2[i][e] = pair(word(kr[i], e));
        acc = ffma2(an2[e], k2[i][e], acc);
        sk[e] = fadd2(sk[e], k2[i][e]);
      }
      float lo, hi;
      f2unpack(acc, lo, hi);
      p[i] = lo + hi;
    }
    // transposing butterfly: 4 partial rows over CH lanes -> one full row dot per lane
    const float u0 = (b1 ? p[2] : p[0]) + __shfl_xor_sync(0xffffffffu, b1 ? p[0] : p[2], B1);
    const float u1 = (b1 ? p[3] : p[1]) + __shfl_xor_sync(0xffffffffu, b1 ? p[1] : p[3], B1);
    float x = (b2 ? u1 : u0) + __shfl_xor_sync(0xffffffffu, b2 ? u0 : u1, B2);
#pragma unroll
    for (int o = B2 / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    x = r + own < r1 ? a.scale * x : -INFINITY;
    float mg = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, B1));
    mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, B2));
    const float mn = fmaxf(m, mg);     // finite: row r is valid
    const float corr = expf(m - mn);   // 0 for the first group
    const float e = expf(x - mn);      // 0 for rows past N
    m = mn;
    float w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = __shfl_sync(0xffffffffu, e, base_lane | ((i & 2) ? B1 : 0) | ((i & 1) ? B2 : 0));
    l = fmaf(l, corr, (w[0] + w[1]) + (w[2] + w[3]));
    const uint64_t c2 = f2pack(corr, corr);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      wk[q] = ffma2(wk[q], c2, 0);
      wv[q] = ffma2(wv[q], c2, 0);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint64_t w2 = f2pack(w[i], w[i]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        wk[q] = ffma2(w2, k2[i][q], wk[q]);
        wv[q] = ffma2(w2, pair(word(vr[i], q)), wv[q]);
      }
    }
    if (r + 4 < r1) load(r + 4, kr, vr);
  }
  // epilogue: normalise, s a.ktil over the head's lanes, write the centroid
  const float inv_n = 1.f / (float)n, inv_l = 1.f / l;
  float mk[8], tk[8], tv[8], pooled = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    f2unpack(sk[q], mk[2 * q], mk[2 * q + 1]);
    f2unpack(wk[q], tk[2 * q], tk[2 * q + 1]);
    f2unpack(wv[q], tv[2 * q], tv[2 * q + 1]);
  }
  float an[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) f2unpack(an2[q], an[2 * q], an[2 * q + 1]);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mk[i] *= inv_n;
    tk[i] *= inv_l;
    tv[i] *= inv_l;
    pooled = fmaf(an[i], tk[i], pooled);
  }
#pragma unroll
  for (int o = CH / 2; o > 0; o >>= 1) pooled += __shfl_xor_sync(0xffffffffu, pooled, o);
  if (!active) return;
  const int64_t row = ((int64_t)b * a.H + h) * a.nb + j;
  float* dst = a.kbar + row * D + c * 8;
  reinterpret_cast<float4*>(dst)[0] = make_float4(mk[0], mk[1], mk[2], mk[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(mk[4], mk[5], mk[6], mk[7]);
  reinterpret_cast<uint4*>(a.kbar16 + row * D + c * 8)[0] =
      make_uint4(pack_bf16x2(tk[0], tk[1]), pack_bf16x2(tk[2], tk[3]), pack_bf16x2(tk[4], tk[5]),
                 pack_bf16x2(tk[6], tk[7]));
  reinterpret_cast<uint4*>(a.vbar16 + row * D + c * 8)[0] =
      make_uint4(pack_bf16x2(tv[0], tv[1]), pack_bf16x2(tv[2], tv[3]), pack_bf16x2(tv[4], tv[5]),
                 pack_bf16x2(tv[6], tv[7]));
  if (c == 0) a.cbias[row] = m + logf(l) - a.scale * pooled;
}

// Residual key codes for INT8 QK (thakicloud "MiniMax-H3 ComfyUI accel stack",
// section 실제 실험 결과, closing accuracy paragraph: only each key block's
// residual from its mean is quantized, the mean term stays bf16).  Per (key
// block, head): kmean16 = the fp32 block mean (kbar, written by the K pass)
// rounded to bf16; r = k - kmean16 in fp32 (a difference of two bf16
// values); sigma = max |r| / 127 over the block's valid rows and all dims;
// codes rint(r * (1 / sigma)) (ties to even, the reciprocal rounded to fp32),
// int8, head-major [B, H, N, D].  Like
// the mean pass, a thread owns 8 dims of one head; the block's rows are read
// twice (the second time from L2): once for the maximum, once for the codes.
template <int D, int HPB>
__global__ void __launch_bounds__(HPB * (D / 8)) quant_k_kernel(const PoolArgs a) {
  constexpr int TPH = D / 8;  // threads per head
  const int j = blockIdx.x;
  const int h = blockIdx.y * HPB + threadIdx.x / TPH;
  const int c = threadIdx.x % TPH;
  const int b = blockIdx.z;
  const bool active = h < a.H;
  const int r0 = j * kBlock, r1 = min(a.N, r0 + kBlock);
  const int64_t row = ((int64_t)b * a.H + h) * a.nb + j;
  const __nv_bfloat16* base = a.src[1] + (int64_t)b * a.sb + (int64_t)h * a.sh + c * 8;
  float m[8];
  if (active) {
    const float4 m0 = *reinterpret_cast<const float4*>(a.kbar + row * D + c * 8);
    const float4 m1 = *reinterpret_cast<const float4*>(a.kbar + row * D + c * 8 + 4);
    const uint4 pk = make_uint4(pack_bf16x2(m0.x, m0.y), pack_bf16x2(m0.z, m0.w), pack_bf16x2(m1.x, m1.y),
                                pack_bf16x2(m1.z, m1.w));
    *reinterpret_cast<uint4*>(a.kmean16 + row * D + c * 8) = pk;
    bf16x8_to_f32(pk, m);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = 0.f;
  }
  float amax = 0.f;
  for (int r = r0; r < r1; r += 8) {
    uint4 u[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      u[k] = make_uint4(0, 0, 0, 0);
      if (active && r + k < r1) u[k] = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)(r + k) * a.sn));
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (r + k < r1) {   // uniform over the CTA
        float f[8];
        bf16x8_to_f32(u[k], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i] - m[i]));
      }
    }
  }
#pragma unroll
  for (int off = TPH / 2; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float sig = amax / 127.f;   // IEEE division (no fast-math)
  const float inv = sig > 0.f ? 1.f / sig : 0.f;
  if (!active) return;
  if (c == 0) a.ksig[row] = sig;
  int8_t* dst = a.kcode + (((int64_t)b * a.H + h) * a.N) * D + c * 8;
  for (int r = r0; r < r1; ++r) {
    const uint4 uk = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)r * a.sn));
    float f[8];
    bf16x8_to_f32(uk, f);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int q = 0;
      if (sig > 0.f) q = min(127, max(-127, __float2int_rn(__fmul_rn(f[i] - m[i], inv))));
      w[i >> 2] |= (uint32_t)(q & 0xff) << (8 * (i & 3));
    }
    *reinterpret_cast<uint2*>(dst + (int64_t)r * D) = make_uint2(w[0], w[1]);
  }
}

// Anchor a = mean of the query rows >= prefix (all rows when prefix >= N),
// from the pooled Q block means (weighted by their row counts) plus the rows
// of the block the prefix ends in.  One CTA per (head, batch) with 1024
// threads: a thread owns a float4 of dims and every G-th block, so the whole
// 2-D sum is in flight in a few rounds; the G partial sums are then added in
// a fixed order (deterministic).
template <int D>
__global__ void __launch_bounds__(1024) anchor_kernel(const __nv_bfloat16* q, int64_t sb, int64_t sn, int64_t sh,
                                                     const float* qbar, int N, int H, int nqb, int prefix,
                                                     float* anchor) {
  constexpr int C4 = D / 4;        // float4 columns of a row
  constexpr int G = 1024 / C4;     // row groups: 32 (D = 128) or 64 (D = 64)
  __shared__ float4 red[G][C4];
  const int h = blockIdx.x, b = blockIdx.y;
  const int c = threadIdx.x % C4, g = threadIdx.x / C4;
  const int P = prefix < N ? prefix : 0;
  const int first = (P + kBlock - 1) / kBlock;   // first block lying wholly at or after P
  const float4* qb = reinterpret_cast<const float4*>(qbar + ((int64_t)b * H + h) * nqb * D) + c;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
  for (int i = first + g; i < nqb; i += G) {
    const float w = (float)(min(N, (i + 1) * kBlock) - i * kBlock);
    const float4 x = qb[(int64_t)i * C4];
    acc.x = fmaf(w, x.x, acc.x);
    acc.y = fmaf(w, x.y, acc.y);
    acc.z = fmaf(w, x.z, acc.z);
    acc.w = fmaf(w, x.w, acc.w);
  }
  // rows [P, first*64) of the block the prefix ends in, read directly
  const __nv_bfloat16* qr = q + (int64_t)b * sb + (int64_t)h * sh + c * 4;
  for (int r = P + g; r < min(N, first * kBlock); r += G) {
    const uint2 u = *reinterpret_cast<const uint2*>(qr + (int64_t)r * sn);
    acc.x += __uint_as_float(u.x << 16);
    acc.y += __uint_as_float(u.x & 0xffff0000u);
    acc.z += __uint_as_float(u.y << 16);
    acc.w += __uint_as_float(u.y & 0xffff0000u);
  }
  red[g][c] = acc;
  __syncthreads();
  if (threadIdx.x < D) {
    const int d = threadIdx.x;
    const float* col = reinterpret_cast<const float*>(&red[0][0]) + d;
    float t = 0.f;
    for (int k = 0; k < G; ++k) t += col[k * D];
    anchor[((int64_t)b * H + h) * D + d] = t / (float)(N - P);
  }
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
    using C = RwCfg<128>;
    dim3 grid(a.nb, (a.H + C::kHeads - 1) / C::kHeads, a.B);
    pool_kv_reweight_kernel<128><<<grid, C::kThreads, 0, st>>>(a);
  } else {
    using C = RwCfg<64>;
    dim3 grid(a.nb, (a.H + C::kHeads - 1) / C::kHeads, a.B);
    pool_kv_reweight_kernel<64><<<grid, C::kThreads, 0, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_k(const PoolArgs& a, int D, cudaStream_t st) {
  if (D != 128) return cudaErrorInvalidValue;
  constexpr int HPB = 8;
  dim3 grid(a.nb, (a.H + HPB - 1) / HPB, a.B);
  quant_k_kernel<128, HPB><<<grid, HPB * 16, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_anchor(const __nv_bfloat16* q, int64_t sb, int64_t sn, int64_t sh, const float* qbar,
                          int B, int N, int H, int D, int nqb, int prefix, float* anchor, cudaStream_t st) {
  dim3 grid(H, B);
  if (D == 128) anchor_kernel<128><<<grid, 1024, 0, st>>>(q, sb, sn, sh, qbar, N, H, nqb, prefix, anchor);
  else anchor_kernel<64><<<grid, 1024, 0, st>>>(q, sb, sn, sh, qbar, N, H, nqb, prefix, anchor);
  return cudaGetLastError();
}

}  // namespace sol
