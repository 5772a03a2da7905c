// Shared definitions of the Sol CUDA path: workspace layout, kernel argument
// blocks, device status word and small PTX helpers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/sol.h"

namespace sol {

constexpr int kBlock = 64;          // rows per query / key block on the GPU path
constexpr int kMaxKeyBlocks = 1024; // ceil(N/64) limit of the routing kernel (N <= 65536)

// Device status word (one per device, owned by the C-ABI layer): kernels set
// it on an expired bounded wait or a bad CSR entry; sol_last_device_status()
// reads and clears it.  The first code raised wins.
__device__ __forceinline__ void raise_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Ints of one query tile's attention plan (built from the CSR lists before the
// attention kernel): a 16-int header (union length, centroid tile count,
// whether the second query block exists, the centroid tiles), both halves'
// exact-block bitmaps (mask_words each), then the union list (<= nkb entries).
__host__ __device__ inline int plan_ints(int mask_words, int nkb) { return (16 + 2 * mask_words + nkb + 3) & ~3; }

// Private workspace layout (byte offsets from the workspace base, 256-aligned).
struct WsLayout {
  int nqb, nkb, mask_words;
  size_t qbar;      // fp32 [B,H,nqb,D]
  size_t kbar;      // fp32 [B,H,nkb,D]
  size_t kbar16;    // bf16 [B,H,nkb,D]
  size_t vbar16;    // bf16 [B,H,nkb,D]
  size_t cbias;     // fp32 [B,H,nkb]  log n_j (+ bias_j)
  size_t anchor;    // fp32 [B,H,D]
  size_t mask;      // uint32 [B*H*nqb, mask_words] exact-block bitmap
  size_t counts;    // int32 [B*H*nqb]
  size_t plan;      // int32 [B*H*ceil(nqb/2)][plan_ints]: per query tile, its attention plan
  size_t kcode;     // int8 [B,H,N,D]  residual key codes (qk_int8 only)
  size_t ksig;      // fp32 [B,H,nkb]  residual scales (qk_int8 only)
  size_t kmean16;   // bf16 [B,H,nkb,D] block means rounded to bf16 (qk_int8 only)
  size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(const sol_params& p) {
  WsLayout L{};
  L.nqb = (p.N + kBlock - 1) / kBlock;
  L.nkb = L.nqb;
  L.mask_words = (L.nkb + 31) / 32;
  size_t bh = (size_t)p.B * p.H, off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  L.qbar = take(bh * L.nqb * p.D * 4);
  L.kbar = take(bh * L.nkb * p.D * 4);
  L.kbar16 = take(bh * L.nkb * p.D * 2);
  L.vbar16 = take(bh * L.nkb * p.D * 2);
  L.cbias = take(bh * L.nkb * 4);
  L.anchor = take(bh * p.D * 4);
  L.mask = take(bh * L.nqb * L.mask_words * 4);
  L.counts = take(bh * L.nqb * 4);
  L.plan = take(bh * ((L.nqb + 1) / 2) * plan_ints(L.mask_words, L.nkb) * 4);
  const size_t i8 = p.qk_int8 ? 1 : 0;
  L.kcode = take(i8 * bh * p.N * p.D);
  L.ksig = take(i8 * bh * L.nkb * 4);
  L.kmean16 = take(i8 * bh * L.nkb * p.D * 2);
  L.total = off;
  return L;
}

template <class T> __host__ __device__ __forceinline__ T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<char*>(base) + off);
}
template <class T> __host__ __device__ __forceinline__ const T* at(const void* base, size_t off) {
  return reinterpret_cast<const T*>(reinterpret_cast<const char*>(base) + off);
}

struct PoolArgs {
  const __nv_bfloat16* src[3];   // q, k, v
  int64_t sb, sn, sh;            // element strides of the inputs
  int B, N, H, nb, prefix;
  float scale;
  int tensor_mask;               // bit t set: pool tensor t in this launch (grid.z = B * popcount)
  int with_bias;                 // K pass also computes the log-mass bias (mean summaries)
  float* qbar; float* kbar; __nv_bfloat16* kbar16; __nv_bfloat16* vbar16;
  float* cbias; const float* anchor;
  int8_t* kcode; float* ksig; __nv_bfloat16* kmean16;   // residual key quantization (qk_int8)
  int* status;                   // device status word (bounded waits)
};

struct RouteArgs {
  const float* qbar; const float* kbar;
  int B, H, N, nqb, nkb, mask_words, n_sink, n_dense;   // n_dense counts the kernel's query rows
  float scale, tau;
  int topk;                      // > 0: Top-K routing keeping topk key blocks (0: threshold)
  int q128;                      // Top-K query rows are 128-row blocks (both 64-row halves share a list)
  uint32_t* mask; int32_t* counts;
  int* status;                   // device status word (bounded waits of the tensor-core scores)
};

struct AttnArgs {
  const __nv_bfloat16* q; const __nv_bfloat16* k; const __nv_bfloat16* v;
  int64_t sb, sn, sh;            // input strides
  __nv_bfloat16* o;
  int64_t ob, on, oh;            // output strides
  float* lse;
  const __nv_bfloat16* kbar16; const __nv_bfloat16* vbar16; const float* cbias;
  const int32_t* row_ptr; const int32_t* col_idx;
  int* plan;                     // workspace region for the per-tile plans
  int B, N, H, nqb, nkb;
  float scale;
  int centroids;                 // 1: a centroid term per unselected key block; 0: unselected blocks dropped
  int qk_int8;                   // 1: exact QK^T from INT8 codes (kcode / ksig / kmean16)
  const int8_t* kcode; const float* ksig; const __nv_bfloat16* kmean16;
  int* status;
};

// Launchers (defined in the kernel files; return the launch error).
cudaError_t launch_pool(const PoolArgs& a, int D, cudaStream_t st);
cudaError_t launch_pool_kv_reweight(const PoolArgs& a, int D, cudaStream_t st);
cudaError_t launch_quant_k(const PoolArgs& a, int D, cudaStream_t st);
cudaError_t launch_anchor(const __nv_bfloat16* q, int64_t sb, int64_t sn, int64_t sh, const float* qbar,
                          int B, int N, int H, int D, int nqb, int prefix, float* anchor, cudaStream_t st);
cudaError_t launch_route(const RouteArgs& a, int D, cudaStream_t st);
cudaError_t launch_scan_compact(const uint32_t* mask, const int32_t* counts, int rows, int mask_words,
                                int32_t* row_ptr, int32_t* col_idx, cudaStream_t st);
cudaError_t launch_attn(const AttnArgs& a, int D, cudaStream_t st);

// Adaptive partition (sol_reblock).  Workspace pieces are caller-owned.
struct ReblockArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  int64_t sb, sn, sh;            // element strides of q and k
  int B, H, N, D;
  int n_fix, n_v;                // rows kept in place (prefix blocks); rows partitioned
  int q_lo, n_q;                 // video query rows [q_lo, q_lo + n_q) of the second moment
  int mchunks;                   // partial-moment chunks per head
  float* mpart;                  // [B*H][mchunks][D][D]
  float* L;                      // [B*H][D][D] lower Cholesky factor
  float* Y;                      // [B*H][n_v][D] whitened unit keys
  int32_t* ord;                  // [B*H][n_v] current order (indices into the partitioned rows)
  int32_t* tmp;                  // [B*H][n_v]
  uint64_t* key;                 // [B*H][n_v] split keys
  int32_t* perm;                 // [B*H][N] output: original row at each position
  int* status;
  int gram_levels;               // top levels whose split axes come from Gram matrices (D = 128)
  float* gpart;                  // Gram partials of one such level: [slots][kGramPartFloats]
  float* wbuf;                   // split axes of one such level: [B*H << lvl][D]
  float* cbuf;                   // [2][B*H << (levels - 1)][D]: group means, the next level's shifts
};
int reblock_levels(int n_v);
int reblock_moment_chunks(int n_q);
int reblock_gram_levels(int n_v, int D);
size_t reblock_gram_part_floats(int BH, int n_v, int D);   // size of ReblockArgs::gpart
size_t reblock_axis_floats(int BH, int n_v, int D);        // size of ReblockArgs::wbuf
cudaError_t launch_reblock(const ReblockArgs& a, int iters, cudaStream_t st);
cudaError_t launch_rows(const int32_t* perm, const __nv_bfloat16* src, __nv_bfloat16* dst, int B, int H, int N, int D,
                        int64_t sb, int64_t sn, int64_t sh, bool gather, int* status, cudaStream_t st);
#ifdef SOL_FAULT_TEST
cudaError_t set_drop_p_arrive(int step);   // fault-test build only
#endif

}  // namespace sol
