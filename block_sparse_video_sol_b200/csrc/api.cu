// C ABI of libsol.so (declared in include/sol.h): argument validation, the
// architecture check, workspace layout and the launch sequence of each stage.
//
// Precedent for the boundary: the Star7 README "MiniMax H3 Activation Chunk &
// Attention Acceleration", section 环境与分发, describes a native library that
// receives only tensor addresses, shapes and the current CUDA stream, does not
// link the PyTorch C++ ABI, and on an architecture mismatch stops with an
// error naming the required and the detected compute capability, with no
// fallback.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace sol {

namespace {

__device__ int g_status = 0;

thread_local char t_err[512] = "";

sol_status fail(sol_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
sol_status fail(sol_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_err, sizeof(t_err), fmt, ap);
  va_end(ap);
  return s;
}

sol_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SOL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Per-device architecture check, done once per device.
constexpr int kMaxDevices = 64;
int g_arch_ok[kMaxDevices];   // 0 unknown, 1 ok, -1 refused
int g_arch_cc[kMaxDevices];
int* g_status_ptr[kMaxDevices];
std::mutex g_arch_mu;

// Checks the current device once and records the device address of its
// status word (the host name of a __device__ variable is not an address).
sol_status check_arch(int** status = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SOL_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_arch_mu);
  if (g_arch_ok[dev] == 0) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    g_arch_cc[dev] = major * 10 + minor;
    g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
    if (g_arch_ok[dev] > 0) {
      void* addr = nullptr;
      e = cudaGetSymbolAddress(&addr, g_status);
      if (e != cudaSuccess) { g_arch_ok[dev] = 0; return cuda_fail(e, "cudaGetSymbolAddress(status)"); }
      g_status_ptr[dev] = static_cast<int*>(addr);
    }
  }
  if (g_arch_ok[dev] < 0)
    return fail(SOL_ERR_UNSUPPORTED, "libsol requires compute capability 10.0 (sm_100a, B200); device %d is %d.%d",
                dev, g_arch_cc[dev] / 10, g_arch_cc[dev] % 10);
  if (status) *status = g_status_ptr[dev];
  return SOL_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape/argument validation shared by every entry point (no CUDA calls).
sol_status validate(const sol_params* p) {
  if (!p) return fail(SOL_ERR_INVALID_ARG, "params is NULL");
  if (p->B < 0 || p->N < 0 || p->H <= 0) return fail(SOL_ERR_INVALID_ARG, "bad shape B=%d N=%d H=%d", p->B, p->N, p->H);
  if (p->D != 64 && p->D != 128) return fail(SOL_ERR_UNSUPPORTED, "head dim %d unsupported (64 or 128)", p->D);
  if (p->routing < 0 || p->routing > 2)
    return fail(SOL_ERR_INVALID_ARG, "routing must be 0 (threshold), 1 (top-k, SLA) or 2 (top-k, compressed branch)");
  const int want_q = p->routing == 1 ? 2 * kBlock : kBlock;
  if (p->q_block != want_q || p->k_block != kBlock)
    return fail(SOL_ERR_UNSUPPORTED, "block sizes %d/%d unsupported (routing %d takes %d/%d)", p->q_block, p->k_block,
                p->routing, want_q, kBlock);
  if (p->routing != 0 && !(p->topk_ratio > 0.f && p->topk_ratio <= 1.f))
    return fail(SOL_ERR_INVALID_ARG, "topk_ratio must lie in (0, 1]");
  if (p->routing == 1 && p->log_mass_bias != 0)
    return fail(SOL_ERR_INVALID_ARG, "top-k routing without the compressed branch has no centroid terms: log_mass_bias must be 0");
  if (p->routing == 0 && (isnan(p->tau) || p->tau == INFINITY))
    return fail(SOL_ERR_INVALID_ARG, "tau must be finite or -inf");
  if (!(p->scale >= 0.f) || isinf(p->scale)) return fail(SOL_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (p->prefix_len < 0 || p->prefix_len > p->N) return fail(SOL_ERR_INVALID_ARG, "prefix_len %d outside [0, N]", p->prefix_len);
  if (p->log_mass_bias < 0 || p->log_mass_bias > 2) return fail(SOL_ERR_INVALID_ARG, "log_mass_bias must be 0, 1 or 2");
  if (p->qk_int8 != 0 && p->qk_int8 != 1) return fail(SOL_ERR_INVALID_ARG, "qk_int8 must be 0 or 1");
  if (p->qk_int8 && p->D != 128) return fail(SOL_ERR_UNSUPPORTED, "qk_int8 needs head dim 128 (got %d)", p->D);
  const int64_t nb = (p->N + kBlock - 1) / kBlock;
  if (nb > kMaxKeyBlocks) return fail(SOL_ERR_UNSUPPORTED, "N=%d exceeds the supported %d rows", p->N, kMaxKeyBlocks * kBlock);
  if ((int64_t)p->B * p->H * nb * nb >= (int64_t)INT32_MAX)
    return fail(SOL_ERR_UNSUPPORTED, "B*H*blocks^2 exceeds int32 CSR indexing");
  const int64_t s[6] = {p->in_stride_b, p->in_stride_n, p->in_stride_h, p->out_stride_b, p->out_stride_n, p->out_stride_h};
  for (int i = 0; i < 6; ++i)
    if (s[i] < 0 || (s[i] & 7)) return fail(SOL_ERR_INVALID_ARG, "stride %lld must be >= 0 and a multiple of 8 elements", (long long)s[i]);
  return SOL_OK;
}

float eff_scale(const sol_params* p) { return p->scale > 0.f ? p->scale : 1.f / sqrtf((float)p->D); }

// Routing kernel arguments shared by sol_route and sol_route_static (the
// caller sets mask and counts).
RouteArgs route_args(const sol_params* p, const WsLayout& L, const void* ws) {
  RouteArgs a{};
  a.qbar = at<float>(ws, L.qbar); a.kbar = at<float>(ws, L.kbar);
  a.B = p->B; a.H = p->H; a.N = p->N; a.nqb = L.nqb; a.nkb = L.nkb; a.mask_words = L.mask_words;
  a.scale = eff_scale(p); a.tau = p->tau;
  a.topk = 0;
  if (p->routing != 0) {
    const double kk = floor((double)p->topk_ratio * (double)L.nkb + 0.5);   // nearest, halves up
    a.topk = (int)std::max(1.0, std::min((double)L.nkb, kk));
  }
  if (p->routing == 1) {   // SLA: 128-row query rows, no KV sink
    a.q128 = 1;
    a.n_sink = 0;
    a.n_dense = (p->prefix_len + 2 * kBlock - 1) / (2 * kBlock);
  } else {                 // threshold, or top-k with the compressed branch
    a.q128 = 0;
    a.n_sink = (p->prefix_len + kBlock - 1) / kBlock;
    a.n_dense = a.n_sink;
  }
  return a;
}
bool empty(const sol_params* p) { return p->B == 0 || p->N == 0; }

}  // namespace
}  // namespace sol

using namespace sol;

extern "C" {

size_t sol_workspace_bytes(const sol_params* p) {
  if (validate(p) != SOL_OK || empty(p)) return 0;
  return ws_layout(*p).total;
}

sol_status sol_workspace_offsets(const sol_params* p, int64_t offsets[8]) {
  sol_status s = validate(p);
  if (s != SOL_OK) return s;
  if (!offsets) return fail(SOL_ERR_INVALID_ARG, "offsets is NULL");
  const WsLayout L = ws_layout(*p);
  const size_t o[8] = {L.qbar, L.kbar, L.kbar16, L.vbar16, L.cbias, L.anchor, L.mask, L.counts};
  for (int i = 0; i < 8; ++i) offsets[i] = (int64_t)o[i];
  return SOL_OK;
}

sol_status sol_workspace_int8_offsets(const sol_params* p, int64_t offsets[3]) {
  sol_status s = validate(p);
  if (s != SOL_OK) return s;
  if (!p->qk_int8) return fail(SOL_ERR_INVALID_ARG, "sol_workspace_int8_offsets: qk_int8 is 0");
  if (!offsets) return fail(SOL_ERR_INVALID_ARG, "offsets is NULL");
  const WsLayout L = ws_layout(*p);
  offsets[0] = (int64_t)L.kcode;
  offsets[1] = (int64_t)L.ksig;
  offsets[2] = (int64_t)L.kmean16;
  return SOL_OK;
}

int64_t sol_col_capacity(const sol_params* p) {
  if (validate(p) != SOL_OK || empty(p)) return 0;
  const int64_t nb = (p->N + kBlock - 1) / kBlock;
  return (int64_t)p->B * p->H * nb * nb;
}

sol_status sol_pool(const sol_params* p, const void* q, const void* k, const void* v, void* ws, size_t ws_bytes,
                    void* stream) {
  sol_status s = validate(p);
  if (s != SOL_OK) return s;
  if (empty(p)) return SOL_OK;
  if (!q || !k || !v || !ws) return fail(SOL_ERR_INVALID_ARG, "sol_pool: NULL pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return fail(SOL_ERR_INVALID_ARG, "sol_pool: q/k/v not 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(SOL_ERR_INVALID_ARG, "sol_pool: workspace not 256-byte aligned");
  const WsLayout L = ws_layout(*p);
  if (ws_bytes < L.total) return fail(SOL_ERR_WORKSPACE, "sol_pool: workspace %zu < %zu bytes", ws_bytes, L.total);
  int* status = nullptr;
  if ((s = check_arch(&status)) != SOL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  PoolArgs a{};
  a.status = status;
  a.src[0] = static_cast<const __nv_bfloat16*>(q);
  a.src[1] = static_cast<const __nv_bfloat16*>(k);
  a.src[2] = static_cast<const __nv_bfloat16*>(v);
  a.sb = p->in_stride_b; a.sn = p->in_stride_n; a.sh = p->in_stride_h;
  a.B = p->B; a.N = p->N; a.H = p->H; a.nb = L.nqb; a.prefix = p->prefix_len;
  a.scale = eff_scale(p);
  a.qbar = at<float>(ws, L.qbar); a.kbar = at<float>(ws, L.kbar);
  a.kbar16 = at<__nv_bfloat16>(ws, L.kbar16); a.vbar16 = at<__nv_bfloat16>(ws, L.vbar16);
  a.cbias = at<float>(ws, L.cbias); a.anchor = at<float>(ws, L.anchor);
  a.kcode = at<int8_t>(ws, L.kcode); a.ksig = at<float>(ws, L.ksig); a.kmean16 = at<__nv_bfloat16>(ws, L.kmean16);
  cudaError_t e;
  if (p->routing == 1) {   // Top-K routing needs no V centroids
    a.tensor_mask = 3; a.with_bias = 0;
    if ((e = launch_pool(a, p->D, st)) != cudaSuccess) return cuda_fail(e, "sol_pool launch");
  } else if (!p->log_mass_bias) {
    a.tensor_mask = 7; a.with_bias = 0;
    if ((e = launch_pool(a, p->D, st)) != cudaSuccess) return cuda_fail(e, "sol_pool launch");
  } else if (p->log_mass_bias == 2) {
    // Q first: the anchor weights the K and V rows of one fused pass.
    a.tensor_mask = 1; a.with_bias = 0;
    if ((e = launch_pool(a, p->D, st)) != cudaSuccess) return cuda_fail(e, "sol_pool launch (q)");
    e = launch_anchor(a.src[0], a.sb, a.sn, a.sh, a.qbar, p->B, p->N, p->H, p->D, L.nqb, p->prefix_len,
                      at<float>(ws, L.anchor), st);
    if (e != cudaSuccess) return cuda_fail(e, "sol_pool anchor launch");
    if ((e = launch_pool_kv_reweight(a, p->D, st)) != cudaSuccess) return cuda_fail(e, "sol_pool launch (k, v reweight)");
  } else {
    // Q (and V) first: the anchor (mean video query) must exist before the K pass.
    a.tensor_mask = 5; a.with_bias = 0;
    if ((e = launch_pool(a, p->D, st)) != cudaSuccess) return cuda_fail(e, "sol_pool launch (q, v)");
    e = launch_anchor(a.src[0], a.sb, a.sn, a.sh, a.qbar, p->B, p->N, p->H, p->D, L.nqb, p->prefix_len,
                      at<float>(ws, L.anchor), st);
    if (e != cudaSuccess) return cuda_fail(e, "sol_pool anchor launch");
    a.tensor_mask = 2; a.with_bias = 1;
    if ((e = launch_pool(a, p->D, st)) != cudaSuccess) return cuda_fail(e, "sol_pool launch (k + bias)");
  }
  if (p->qk_int8 && (e = launch_quant_k(a, p->D, st)) != cudaSuccess) return cuda_fail(e, "sol_pool launch (k residual codes)");
  return SOL_OK;
}

sol_status sol_route(const sol_params* p, void* ws, size_t ws_bytes, int32_t* row_ptr, int32_t* col_idx, void* stream) {
  sol_status s = validate(p);
  if (s != SOL_OK) return s;
  if (empty(p)) return SOL_OK;
  if (!ws || !row_ptr || !col_idx) return fail(SOL_ERR_INVALID_ARG, "sol_route: NULL pointer");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(SOL_ERR_INVALID_ARG, "sol_route: workspace not 256-byte aligned");
  const WsLayout L = ws_layout(*p);
  if (ws_bytes < L.total) return fail(SOL_ERR_WORKSPACE, "sol_route: workspace %zu < %zu bytes", ws_bytes, L.total);
  int* status = nullptr;
  if ((s = check_arch(&status)) != SOL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RouteArgs a = route_args(p, L, ws);
  a.mask = at<uint32_t>(ws, L.mask); a.counts = at<int32_t>(ws, L.counts);
  a.status = status;
  cudaError_t e = launch_route(a, p->D, st);
  if (e != cudaSuccess) return cuda_fail(e, "sol_route launch");
  e = launch_scan_compact(a.mask, a.counts, p->B * p->H * L.nqb, L.mask_words, row_ptr, col_idx, st);
  if (e != cudaSuccess) return cuda_fail(e, "sol_route scan/compact launch");
  return SOL_OK;
}

sol_status sol_attn_fwd(const sol_params* p, const void* q, const void* k, const void* v, const void* ws,
                        size_t ws_bytes, const int32_t* row_ptr, const int32_t* col_idx, void* o, float* lse,
                        void* stream) {
  sol_status s = validate(p);
  if (s != SOL_OK) return s;
  if (empty(p)) return SOL_OK;
  if (!q || !k || !v || !ws || !row_ptr || !col_idx || !o) return fail(SOL_ERR_INVALID_ARG, "sol_attn_fwd: NULL pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(SOL_ERR_INVALID_ARG, "sol_attn_fwd: q/k/v/o not 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(SOL_ERR_INVALID_ARG, "sol_attn_fwd: workspace not 256-byte aligned");
  const WsLayout L = ws_layout(*p);
  if (ws_bytes < L.total) return fail(SOL_ERR_WORKSPACE, "sol_attn_fwd: workspace %zu < %zu bytes", ws_bytes, L.total);
  int* status = nullptr;
  if ((s = check_arch(&status)) != SOL_OK) return s;
  AttnArgs a{};
  a.status = status;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.sb = p->in_stride_b; a.sn = p->in_stride_n; a.sh = p->in_stride_h;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.ob = p->out_stride_b; a.on = p->out_stride_n; a.oh = p->out_stride_h;
  a.lse = lse;
  a.kbar16 = at<__nv_bfloat16>(ws, L.kbar16); a.vbar16 = at<__nv_bfloat16>(ws, L.vbar16);
  a.cbias = at<float>(ws, L.cbias);
  a.row_ptr = row_ptr; a.col_idx = col_idx;
  a.plan = at<int>(const_cast<void*>(ws), L.plan);
  a.B = p->B; a.N = p->N; a.H = p->H; a.nqb = L.nqb; a.nkb = L.nkb;
  a.scale = eff_scale(p);
  a.centroids = p->routing == 1 ? 0 : 1;
  a.qk_int8 = p->qk_int8;
  a.kcode = at<int8_t>(ws, L.kcode); a.ksig = at<float>(ws, L.ksig); a.kmean16 = at<__nv_bfloat16>(ws, L.kmean16);
  cudaError_t e = launch_attn(a, p->D, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "sol_attn_fwd launch");
  return SOL_OK;
}

sol_status sol_last_device_status(void* stream) {
  sol_status s0 = check_arch();
  if (s0 != SOL_OK) return s0;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, g_status, sizeof(int));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "device status read");
  if (v == 0) return SOL_OK;
  return fail((sol_status)v, "device status: %s", sol_status_string((sol_status)v));
}

// ---- adaptive partition (Spark-Reblock reading) and row gathers ------------------------------
namespace {
struct ReblockLayout {
  int n_fix, n_v, q_lo, n_q, mchunks;
  size_t mpart, L, Y, ord, tmp, key, gpart, wbuf, cbuf, total;
};
ReblockLayout reblock_layout(const sol_params& p) {
  ReblockLayout R{};
  const int nsink = (p.prefix_len + kBlock - 1) / kBlock;
  R.n_fix = std::min(p.N, kBlock * nsink);
  R.n_v = p.N - R.n_fix;
  R.q_lo = p.prefix_len < p.N ? p.prefix_len : 0;   // the video query rows (all rows if none)
  R.n_q = p.N - R.q_lo;
  R.mchunks = R.n_q > 0 ? reblock_moment_chunks(R.n_q) : 0;
  const size_t bh = (size_t)p.B * p.H, D = p.D;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  // the partial moments are dead once L is factored: the levels' Gram partials reuse them
  R.mpart = take(std::max(bh * R.mchunks * D * D, reblock_gram_part_floats((int)bh, R.n_v, p.D)) * 4);
  R.gpart = R.mpart;
  R.L = take(bh * D * D * 4);
  R.Y = take(bh * R.n_v * D * 4);
  R.ord = take(bh * R.n_v * 4);
  R.tmp = take(bh * R.n_v * 4);
  R.key = take(bh * R.n_v * 8);
  R.wbuf = take(reblock_axis_floats((int)bh, R.n_v, p.D) * 4);
  R.cbuf = take(2 * reblock_axis_floats((int)bh, R.n_v, p.D) * 4);
  R.total = R.n_v > 0 ? off : 0;
  return R;
}
constexpr int kReblockIters = 4;   // power steps per split
}  // namespace

size_t sol_reblock_workspace_bytes(const sol_params* p) {
  if (validate(p) != SOL_OK || empty(p)) return 0;
  return reblock_layout(*p).total;
}

sol_status sol_reblock(const sol_params* p, const void* q, const void* k, void* ws, size_t ws_bytes, int32_t* perm,
                       void* stream) {
  sol_status s = validate(p);
  if (s != SOL_OK) return s;
  if (empty(p)) return SOL_OK;
  if (!q || !k || !perm) return fail(SOL_ERR_INVALID_ARG, "sol_reblock: NULL pointer");
  if (!aligned16(q) || !aligned16(k)) return fail(SOL_ERR_INVALID_ARG, "sol_reblock: q/k not 16-byte aligned");
  const ReblockLayout R = reblock_layout(*p);
  if (R.total > 0) {
    if (!ws) return fail(SOL_ERR_INVALID_ARG, "sol_reblock: NULL workspace");
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
      return fail(SOL_ERR_INVALID_ARG, "sol_reblock: workspace not 256-byte aligned");
    if (ws_bytes < R.total) return fail(SOL_ERR_WORKSPACE, "sol_reblock: workspace %zu < %zu bytes", ws_bytes, R.total);
  }
  int* status = nullptr;
  if ((s = check_arch(&status)) != SOL_OK) return s;
  ReblockArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.sb = p->in_stride_b; a.sn = p->in_stride_n; a.sh = p->in_stride_h;
  a.B = p->B; a.H = p->H; a.N = p->N; a.D = p->D;
  a.n_fix = R.n_fix; a.n_v = R.n_v; a.q_lo = R.q_lo; a.n_q = R.n_q; a.mchunks = R.mchunks;
  if (R.total > 0) {
    a.mpart = at<float>(ws, R.mpart); a.L = at<float>(ws, R.L); a.Y = at<float>(ws, R.Y);
    a.ord = at<int32_t>(ws, R.ord); a.tmp = at<int32_t>(ws, R.tmp); a.key = at<uint64_t>(ws, R.key);
    a.gpart = at<float>(ws, R.gpart); a.wbuf = at<float>(ws, R.wbuf); a.cbuf = at<float>(ws, R.cbuf);
  }
  a.gram_levels = reblock_gram_levels(R.n_v, p->D);
  a.perm = perm;
  a.status = status;
  const cudaError_t e = launch_reblock(a, kReblockIters, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "sol_reblock launch");
  return SOL_OK;
}

static sol_status rows_entry(const sol_params* p, const int32_t* perm, const void* src, void* dst, bool gather,
                             void* stream, const char* name) {
  sol_status s = validate(p);
  if (s != SOL_OK) return s;
  if (empty(p)) return SOL_OK;
  if (!perm || !src || !dst) return fail(SOL_ERR_INVALID_ARG, "%s: NULL pointer", name);
  if (!aligned16(src) || !aligned16(dst)) return fail(SOL_ERR_INVALID_ARG, "%s: tensors not 16-byte aligned", name);
  int* status = nullptr;
  if ((s = check_arch(&status)) != SOL_OK) return s;
  const int64_t sb = gather ? p->in_stride_b : p->out_stride_b, sn = gather ? p->in_stride_n : p->out_stride_n,
                sh = gather ? p->in_stride_h : p->out_stride_h;
  const cudaError_t e = launch_rows(perm, static_cast<const __nv_bfloat16*>(src), static_cast<__nv_bfloat16*>(dst), p->B,
                                    p->H, p->N, p->D, sb, sn, sh, gather, status, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, name);
  return SOL_OK;
}

sol_status sol_gather_rows(const sol_params* p, const int32_t* perm, const void* x, void* xp, void* stream) {
  return rows_entry(p, perm, x, xp, true, stream, "sol_gather_rows");
}

sol_status sol_scatter_rows(const sol_params* p, const int32_t* perm, const void* xp, void* x, void* stream) {
  return rows_entry(p, perm, xp, x, false, stream, "sol_scatter_rows");
}

sol_status sol_debug_drop_arrive(int32_t step) {
#ifdef SOL_FAULT_TEST
  sol_status s = check_arch();
  if (s != SOL_OK) return s;
  if (step < -1) return fail(SOL_ERR_INVALID_ARG, "sol_debug_drop_arrive: step %d < -1", (int)step);
  const cudaError_t e = sol::set_drop_p_arrive(step);
  if (e != cudaSuccess) return cuda_fail(e, "sol_debug_drop_arrive");
  return SOL_OK;
#else
  (void)step;
  return fail(SOL_ERR_UNSUPPORTED, "sol_debug_drop_arrive: this library was built without SOL_FAULT_TEST");
#endif
}

const char* sol_status_string(sol_status s) {
  switch (s) {
    case SOL_OK: return "SOL_OK";
    case SOL_ERR_INVALID_ARG: return "SOL_ERR_INVALID_ARG";
    case SOL_ERR_UNSUPPORTED: return "SOL_ERR_UNSUPPORTED";
    case SOL_ERR_WORKSPACE: return "SOL_ERR_WORKSPACE";
    case SOL_ERR_CUDA: return "SOL_ERR_CUDA";
    case SOL_ERR_TIMEOUT: return "SOL_ERR_TIMEOUT";
  }
  return "SOL_ERR_UNKNOWN";
}

const char* sol_last_error_text(void) { return t_err; }

}  // extern "C"

// ---------------------------------------------------------------------------
// sol_route_static: sol_route for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand the library extra device
// buffers: a host framework that owns every device allocation through its
// own fixed-budget pool, or a code path that must not allocate (allocation
// can synchronise the device or fail at an inconvenient time).  For them this
// entry point keeps sol_route's scratch -- the exact-block bitmap and the
// per-row counts -- in one fixed array inside the library, so the caller only
// provides the pooled input (the workspace sol_pool filled, of which only the
// part before the bitmap is read) and the CSR outputs.
//
// The array holds kRouteScratchBytes (8 MiB); every GPU that loads the
// library keeps it until the process exits.  A problem needs
// B*H*ceil(N/64)*ceil(ceil(N/64)/32)*4 bytes of bitmap (rounded up to 256)
// plus B*H*ceil(N/64)*4 bytes of counts; larger problems are rejected with
// SOL_ERR_UNSUPPORTED.  Every call shares the array and it keeps the last
// call's contents; each call writes every bitmap word and count it later
// reads, so nothing needs clearing.  Calls whose executions overlap on the GPU
// (different streams, or different host threads, on one device) race on the
// array.  The first call on a device looks up the array's device address
// (cudaGetSymbolAddress) and caches it; make that first call before any
// stream capture.
static constexpr size_t kRouteScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char sol_route_scratch[kRouteScratchBytes];

namespace sol {
namespace {

unsigned char* g_route_scratch_ptr[kMaxDevices];
std::mutex g_route_scratch_mu;

// Device address of this device's copy of the array (the host-side name of a
// __device__ variable is only a stand-in, never a device address).
sol_status route_scratch(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SOL_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_route_scratch_mu);
  if (!g_route_scratch_ptr[dev]) {
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, sol_route_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(route scratch)");
    g_route_scratch_ptr[dev] = static_cast<unsigned char*>(addr);
  }
  *out = g_route_scratch_ptr[dev];
  return SOL_OK;
}

}  // namespace
}  // namespace sol

extern "C" sol_status sol_route_static(const sol_params* p, const void* ws, size_t ws_bytes, int32_t* row_ptr,
                                       int32_t* col_idx, void* stream) {
  sol_status s = validate(p);
  if (s != SOL_OK) return s;
  if (empty(p)) return SOL_OK;
  if (!ws || !row_ptr || !col_idx) return fail(SOL_ERR_INVALID_ARG, "sol_route_static: NULL pointer");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(SOL_ERR_INVALID_ARG, "sol_route_static: workspace not 256-byte aligned");
  const WsLayout L = ws_layout(*p);
  if (ws_bytes < L.mask)
    return fail(SOL_ERR_WORKSPACE, "sol_route_static: pooled workspace %zu < %zu bytes", ws_bytes, L.mask);
  const size_t rows = (size_t)p->B * p->H * L.nqb;
  const size_t mask_bytes = align256(rows * L.mask_words * 4);
  const size_t need = mask_bytes + rows * 4;
  if (need > kRouteScratchBytes)
    return fail(SOL_ERR_UNSUPPORTED,
                "sol_route_static: this problem needs %zu bytes of routing scratch; the built-in array holds %zu "
                "(use sol_route with a caller-allocated workspace)", need, kRouteScratchBytes);
  int* status = nullptr;
  if ((s = check_arch(&status)) != SOL_OK) return s;
  unsigned char* scratch = nullptr;
  if ((s = route_scratch(&scratch)) != SOL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RouteArgs a = route_args(p, L, ws);
  a.mask = reinterpret_cast<uint32_t*>(scratch);
  a.counts = reinterpret_cast<int32_t*>(scratch + mask_bytes);
  a.status = status;
  cudaError_t e = launch_route(a, p->D, st);
  if (e != cudaSuccess) return cuda_fail(e, "sol_route_static launch");
  e = launch_scan_compact(a.mask, a.counts, (int)rows, L.mask_words, row_ptr, col_idx, st);
  if (e != cudaSuccess) return cuda_fail(e, "sol_route_static scan/compact launch");
  return SOL_OK;
}

// ---------------------------------------------------------------------------
// sol_forward_host: the whole forward pass on host buffers.
//
// Heads are independent in every stage, so the call splits them into chunks
// of heads_per_chunk heads and pipelines them through two staging slots in
// the caller's device buffer: the copy of chunk c+1's Q/K/V into one slot
// (a copy-in stream) overlaps chunk c's pool/route/attention on the caller's
// stream, which overlaps chunk c-1's O copy back to the host (a copy-out
// stream).  Host->device and device->host copies run on different copy
// engines, so the call takes about the time of its host->device bytes plus
// one chunk's compute and copy-out.  Host rows are gathered with strided 2-D
// copies (one per batch element, or per head when heads are not adjacent).
// Results are those of sol_pool + sol_route + sol_attn_fwd on the whole
// problem, bit for bit (every stage is per head).
namespace sol {
namespace {

struct HostLayout {
  sol_params cp;   // a full chunk: hc heads, compact [B, N, hc, D] strides
  size_t q, k, v, o, ws, row_ptr, col_idx, slot;
};
constexpr int kHostSlots = 2;
constexpr int kDefaultHeadsPerChunk = 4;   // measured at H=56, N=32768: 27.5 ms per step against 27.8 (2), 28.5 (8), 31.6 (14)

HostLayout host_layout(const sol_params* p, int hc) {
  HostLayout L{};
  L.cp = *p;
  L.cp.H = hc;
  const int64_t rowe = (int64_t)hc * p->D;
  L.cp.in_stride_b = L.cp.out_stride_b = (int64_t)p->N * rowe;
  L.cp.in_stride_n = L.cp.out_stride_n = rowe;
  L.cp.in_stride_h = L.cp.out_stride_h = p->D;
  const size_t tb = (size_t)p->B * p->N * rowe * 2;
  const size_t nb = (size_t)(p->N + kBlock - 1) / kBlock;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  L.q = take(tb); L.k = take(tb); L.v = take(tb); L.o = take(tb);
  L.ws = take(ws_layout(L.cp).total);
  L.row_ptr = take(((size_t)p->B * hc * nb + 1) * 4);
  L.col_idx = take((size_t)p->B * hc * nb * nb * 4);
  L.slot = off;
  return L;
}

int heads_per_chunk(const sol_params* p, int32_t hc) {
  return std::min(p->H, hc > 0 ? hc : kDefaultHeadsPerChunk);
}

// Per-device copy streams and events, created on first use and kept until
// exit.  The enqueue phase of a call holds the mutex, so calls from several
// host threads use the events one after the other.
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t entry = nullptr, ev_in[kHostSlots] = {}, ev_comp[kHostSlots] = {}, ev_out[kHostSlots] = {};
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mu;

sol_status host_pipe(HostPipe** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SOL_ERR_UNSUPPORTED, "device index %d out of range", dev);
  HostPipe& P = g_pipe[dev];
  if (!P.in) {
    const unsigned ef = cudaEventDisableTiming;
    e = cudaStreamCreateWithFlags(&P.in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&P.out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&P.entry, ef);
    for (int s = 0; s < kHostSlots && e == cudaSuccess; ++s) {
      e = cudaEventCreateWithFlags(&P.ev_in[s], ef);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&P.ev_comp[s], ef);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&P.ev_out[s], ef);
    }
    if (e != cudaSuccess) { P.in = nullptr; return cuda_fail(e, "sol_forward_host: stream/event creation"); }
  }
  *out = &P;
  return SOL_OK;
}

// Strided 2-D copy of nh heads x D of every row of B x N rows between a
// host tensor (strides sb, sn, sh in elements) and a compact device chunk.
cudaError_t copy_chunk(void* dev, void* host, int64_t sb, int64_t sn, int64_t sh, int B, int N, int nh, int D,
                       int64_t rowe, bool to_dev, cudaStream_t st) {
  const cudaMemcpyKind kind = to_dev ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost;
  const size_t hpitch = (size_t)sn * 2, dpitch = (size_t)rowe * 2;
  const int groups = sh == D ? 1 : nh;   // adjacent heads go in one copy
  const size_t width = (size_t)(sh == D ? nh : 1) * D * 2;
  for (int b = 0; b < B; ++b)
    for (int g = 0; g < groups; ++g) {
      char* h = static_cast<char*>(host) + ((int64_t)b * sb + (int64_t)g * sh) * 2;
      char* d = static_cast<char*>(dev) + ((int64_t)b * N * rowe + (int64_t)g * D) * 2;
      const cudaError_t e = to_dev ? cudaMemcpy2DAsync(d, dpitch, h, hpitch, width, N, kind, st)
                                   : cudaMemcpy2DAsync(h, hpitch, d, dpitch, width, N, kind, st);
      if (e != cudaSuccess) return e;
    }
  return cudaSuccess;
}

}  // namespace
}  // namespace sol

extern "C" size_t sol_host_staging_bytes(const sol_params* p, int32_t hc) {
  if (validate(p) != SOL_OK || empty(p) || hc < 0) return 0;
  return kHostSlots * host_layout(p, heads_per_chunk(p, hc)).slot;
}

extern "C" sol_status sol_forward_host(const sol_params* p, const void* q, const void* k, const void* v, void* o,
                                       int32_t hc_req, void* staging, size_t staging_bytes, void* stream) {
  sol_status s = validate(p);
  if (s != SOL_OK) return s;
  if (empty(p)) return SOL_OK;
  if (hc_req < 0) return fail(SOL_ERR_INVALID_ARG, "sol_forward_host: heads_per_chunk must be >= 0");
  if (!q || !k || !v || !o || !staging) return fail(SOL_ERR_INVALID_ARG, "sol_forward_host: NULL pointer");
  if ((reinterpret_cast<uintptr_t>(staging) & 255u) != 0)
    return fail(SOL_ERR_INVALID_ARG, "sol_forward_host: staging not 256-byte aligned");
  const int hc = heads_per_chunk(p, hc_req);
  const HostLayout L = host_layout(p, hc);
  if (staging_bytes < kHostSlots * L.slot)
    return fail(SOL_ERR_WORKSPACE, "sol_forward_host: staging %zu < %zu bytes", staging_bytes, kHostSlots * L.slot);
  if ((s = check_arch()) != SOL_OK) return s;
  std::lock_guard<std::mutex> lk(g_pipe_mu);
  HostPipe* P = nullptr;
  if ((s = host_pipe(&P)) != SOL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t rowe = (int64_t)hc * p->D;
  const int chunks = (p->H + hc - 1) / hc;
  cudaError_t e;
  // earlier work on the caller's stream (a previous call on this staging) comes first
  if ((e = cudaEventRecord(P->entry, st)) != cudaSuccess) return cuda_fail(e, "sol_forward_host: event record");
  if ((e = cudaStreamWaitEvent(P->in, P->entry, 0)) != cudaSuccess) return cuda_fail(e, "sol_forward_host: wait");
  for (int c = 0; c < chunks; ++c) {
    const int slot = c % kHostSlots, h0 = c * hc, nh = std::min(hc, p->H - h0);
    char* base = static_cast<char*>(staging) + (size_t)slot * L.slot;
    sol_params cp = L.cp;
    cp.H = nh;
    // copy in (after the compute that last read this slot)
    if (c >= kHostSlots && (e = cudaStreamWaitEvent(P->in, P->ev_comp[slot], 0)) != cudaSuccess)
      return cuda_fail(e, "sol_forward_host: wait");
    const void* src[3] = {q, k, v};
    const size_t dst[3] = {L.q, L.k, L.v};
    for (int t = 0; t < 3; ++t) {
      e = copy_chunk(base + dst[t], const_cast<char*>(static_cast<const char*>(src[t])) + (int64_t)h0 * p->in_stride_h * 2,
                     p->in_stride_b, p->in_stride_n, p->in_stride_h, p->B, p->N, nh, p->D, rowe, true, P->in);
      if (e != cudaSuccess) return cuda_fail(e, "sol_forward_host: host-to-device copy");
    }
    if ((e = cudaEventRecord(P->ev_in[slot], P->in)) != cudaSuccess) return cuda_fail(e, "sol_forward_host: event record");
    // compute on the caller's stream (after the copy-out that last read this slot's O)
    if ((e = cudaStreamWaitEvent(st, P->ev_in[slot], 0)) != cudaSuccess) return cuda_fail(e, "sol_forward_host: wait");
    if (c >= kHostSlots && (e = cudaStreamWaitEvent(st, P->ev_out[slot], 0)) != cudaSuccess)
      return cuda_fail(e, "sol_forward_host: wait");
    const size_t wsb = ws_layout(cp).total;
    int32_t* rp = reinterpret_cast<int32_t*>(base + L.row_ptr);
    int32_t* ci = reinterpret_cast<int32_t*>(base + L.col_idx);
    if ((s = sol_pool(&cp, base + L.q, base + L.k, base + L.v, base + L.ws, wsb, stream)) != SOL_OK) return s;
    if ((s = sol_route(&cp, base + L.ws, wsb, rp, ci, stream)) != SOL_OK) return s;
    if ((s = sol_attn_fwd(&cp, base + L.q, base + L.k, base + L.v, base + L.ws, wsb, rp, ci, base + L.o, nullptr,
                          stream)) != SOL_OK)
      return s;
    if ((e = cudaEventRecord(P->ev_comp[slot], st)) != cudaSuccess) return cuda_fail(e, "sol_forward_host: event record");
    // copy out
    if ((e = cudaStreamWaitEvent(P->out, P->ev_comp[slot], 0)) != cudaSuccess) return cuda_fail(e, "sol_forward_host: wait");
    e = copy_chunk(base + L.o, static_cast<char*>(o) + (int64_t)h0 * p->out_stride_h * 2, p->out_stride_b,
                   p->out_stride_n, p->out_stride_h, p->B, p->N, nh, p->D, rowe, false, P->out);
    if (e != cudaSuccess) return cuda_fail(e, "sol_forward_host: device-to-host copy");
    if ((e = cudaEventRecord(P->ev_out[slot], P->out)) != cudaSuccess) return cuda_fail(e, "sol_forward_host: event record");
  }
  // the caller's stream completes only after every chunk's O is on the host
  for (int slot = 0; slot < std::min(chunks, kHostSlots); ++slot)
    if ((e = cudaStreamWaitEvent(st, P->ev_out[slot], 0)) != cudaSuccess) return cuda_fail(e, "sol_forward_host: wait");
  return SOL_OK;
}
