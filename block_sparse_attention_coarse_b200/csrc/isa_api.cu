// Host implementation of the C interface declared in include/isa.h:
// argument checks, plan-workspace layout, TMA tensor maps and launches.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "isa_common.cuh"

using namespace isa;

namespace {

thread_local std::string g_last_error = "no error";
// process-wide settings, read by every launch (any host thread may set them)
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<int> g_inject{0};

isa_status fail(isa_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
isa_status fail(isa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

isa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(ISA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

isa_status make_dims(const isa_params* p, Dims* dm) {
  if (!p) return fail(ISA_ERR_INVALID_ARG, "params is NULL");
  if (p->B <= 0 || p->H <= 0 || p->L_src <= 0 || p->L_ctx <= 0 || p->block <= 0 || p->D <= 0)
    return fail(ISA_ERR_INVALID_ARG, "B, H, D, L_src, L_ctx and block must be positive");
  if (!(p->alpha_s > 0.f && p->alpha_s <= 1.f))
    return fail(ISA_ERR_INVALID_ARG, "alpha_s must lie in (0, 1], got %g", (double)p->alpha_s);
  if (!(p->alpha_f >= 0.f && p->alpha_f <= 1.f))
    return fail(ISA_ERR_INVALID_ARG, "alpha_f must lie in [0, 1], got %g", (double)p->alpha_f);
  if (!(p->alpha_ns >= 0.f && p->alpha_ns <= 1.f))
    return fail(ISA_ERR_INVALID_ARG, "alpha_ns must lie in [0, 1], got %g", (double)p->alpha_ns);
  if (std::isnan(p->scale) || std::isinf(p->scale)) return fail(ISA_ERR_INVALID_ARG, "scale must be finite");
  if (p->D != 64 && p->D != 128) return fail(ISA_ERR_UNSUPPORTED, "D must be 64 or 128, got %d", p->D);
  if (p->block != 32 && p->block != 64) return fail(ISA_ERR_UNSUPPORTED, "block must be 32 or 64, got %d", p->block);
  const long long L = (long long)p->L_src + p->L_ctx;
  const long long BH = (long long)p->B * p->H;
  if (BH * L * p->D >= (1ll << 31) || BH * L >= (1ll << 31))
    return fail(ISA_ERR_UNSUPPORTED, "B*H*L*D must stay below 2^31");
  Dims d{};
  d.B = p->B;
  d.H = p->H;
  d.BH = (int)BH;
  d.D = p->D;
  d.L_src = p->L_src;
  d.L_ctx = p->L_ctx;
  d.L = (int)L;
  d.b = p->block;
  d.T_src = (p->L_src + d.b - 1) / d.b;
  d.T_ctx = (p->L_ctx + d.b - 1) / d.b;
  d.T = d.T_src + d.T_ctx;
  if (d.T > kMaxT) return fail(ISA_ERR_UNSUPPORTED, "at most %d blocks per head, got %d", kMaxT, d.T);
  // counts from the float32 ratios, evaluated in double
  const double as = (double)p->alpha_s, af = (double)p->alpha_f, ans = (double)p->alpha_ns;
  long long ks = (long long)std::ceil(as * d.T_ctx);
  d.K_sel = (int)std::min<long long>(std::max<long long>(ks, 1), d.T_ctx);
  d.T_kv = d.T_src + d.K_sel;
  if (d.T_kv > kMaxTkv) return fail(ISA_ERR_UNSUPPORTED, "at most %d kept blocks per head, got %d", kMaxTkv, d.T_kv);
  long long nf = (long long)std::floor(af * d.T);
  d.n_flat = (int)std::min<long long>(std::max<long long>(nf, 0), d.T);
  d.n_sharp = d.T - d.n_flat;
  long long ne = (long long)std::ceil(ans * d.T_kv);
  d.n_exact = (int)std::min<long long>(std::max<long long>(ne, 0), d.T_kv);
  d.T_kv_pad = (d.T_kv + 127) / 128 * 128;
  d.words = (d.T_kv + 31) / 32;
  d.scale = p->scale > 0.f ? p->scale : (float)(1.0 / std::sqrt((double)p->D));
  *dm = d;
  return ISA_OK;
}

PlanLayout make_layout(const Dims& d) {
  PlanLayout L{};
  size_t off = 0;
  auto put = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t BH = d.BH;
  L.status = put(256);
  L.Qc = put(BH * d.T * d.D * 4);
  L.Kc = put(BH * d.T * d.D * 4);
  L.Vc = put(BH * d.T * d.D * 4);
  L.imp = put(BH * d.T_ctx * 4);
  L.ctx_sel = put(BH * d.K_sel * 4);
  L.kept = put(BH * d.T_kv * 4);
  L.energy = put(BH * d.T * 4);
  L.sharp = put(BH * std::max(d.n_sharp, 1) * 4);
  L.flat = put(BH * std::max(d.n_flat, 1) * 4);
  L.exact = put(BH * std::max(d.n_flat, 1) * std::max(d.n_exact, 1) * 4);
  L.bits = put(BH * std::max(d.n_flat, 1) * d.words * 4);
  L.Kp = put(BH * d.T_kv_pad * d.D * 2);
  L.Vp = put(BH * d.T_kv_pad * d.D * 2);
  L.total = off;
  return L;
}

PlanPtrs make_ptrs(const PlanLayout& L, void* ws) {
  char* b = static_cast<char*>(ws);
  PlanPtrs p;
  p.status = reinterpret_cast<int*>(b + L.status);
  p.Qc = reinterpret_cast<float*>(b + L.Qc);
  p.Kc = reinterpret_cast<float*>(b + L.Kc);
  p.Vc = reinterpret_cast<float*>(b + L.Vc);
  p.imp = reinterpret_cast<float*>(b + L.imp);
  p.ctx_sel = reinterpret_cast<int*>(b + L.ctx_sel);
  p.kept = reinterpret_cast<int*>(b + L.kept);
  p.energy = reinterpret_cast<float*>(b + L.energy);
  p.sharp = reinterpret_cast<int*>(b + L.sharp);
  p.flat = reinterpret_cast<int*>(b + L.flat);
  p.exact = reinterpret_cast<int*>(b + L.exact);
  p.bits = reinterpret_cast<uint32_t*>(b + L.bits);
  p.Kp = reinterpret_cast<__nv_bfloat16*>(b + L.Kp);
  p.Vp = reinterpret_cast<__nv_bfloat16*>(b + L.Vp);
  return p;
}

isa_status check_ptr(const void* p, const char* name, size_t align) {
  if (!p) return fail(ISA_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % align) return fail(ISA_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
  return ISA_OK;
}

// ---- driver entry point for tensor-map encoding (no link against libcuda) ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_once;
cudaError_t g_init_err = cudaSuccess;

void init_once() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  g_init_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (g_init_err == cudaSuccess && q != cudaDriverEntryPointSuccess) g_init_err = cudaErrorNotSupported;
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
}

isa_status ensure_init() {
  std::call_once(g_once, init_once);
  if (g_init_err != cudaSuccess || !g_encode) return cuda_fail(g_init_err, "library initialisation");
  return ISA_OK;
}

}  // namespace

namespace isa {
// Makes the device that owns `ptr` current on the calling thread (binding its
// primary context), so that a call from a thread that never selected a
// device -- a framework's autograd worker, a thread pool -- encodes its
// tensor maps and launches on the GPU that holds the data.
isa_status bind_device_of(const void* ptr, const char* name) {
  cudaPointerAttributes at{};
  cudaError_t e = cudaPointerGetAttributes(&at, ptr);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, name);
  }
  if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
    return fail(ISA_ERR_INVALID_ARG, "%s is not CUDA device memory", name);
  if ((e = cudaSetDevice(at.device)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  return ISA_OK;
}
}  // namespace isa

namespace {

// rows x D bf16, box of 64 columns x box_rows rows, 128-byte swizzle
isa_status make_map(CUtensorMap* m, const void* base, uint64_t rows, int D, int box_rows, const char* name) {
  cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ISA_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with %d", name, (int)r);
  return ISA_OK;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace

namespace isa {
// Sets the calling thread's isa_last_error() text (used by other files of the
// library that report their own errors).
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace isa

extern "C" {

isa_status isa_plan_workspace_size(const isa_params* p, size_t* bytes) {
  if (!bytes) return fail(ISA_ERR_INVALID_ARG, "bytes is NULL");
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  *bytes = make_layout(d).total;
  return ISA_OK;
}

isa_status isa_plan_view_get(const isa_params* p, const void* ws, size_t ws_bytes, isa_plan_view* v) {
  if (!v) return fail(ISA_ERR_INVALID_ARG, "view is NULL");
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  if ((s = check_ptr(ws, "workspace", 256)) != ISA_OK) return s;
  const PlanLayout L = make_layout(d);
  if (ws_bytes < L.total) return fail(ISA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  const PlanPtrs pp = make_ptrs(L, const_cast<void*>(ws));
  v->T_src = d.T_src;
  v->T_ctx = d.T_ctx;
  v->T = d.T;
  v->K_sel = d.K_sel;
  v->T_kv = d.T_kv;
  v->n_flat = d.n_flat;
  v->n_sharp = d.n_sharp;
  v->n_exact = d.n_exact;
  v->T_kv_pad = d.T_kv_pad;
  v->bitmap_words = d.words;
  v->Qc = pp.Qc;
  v->Kc = pp.Kc;
  v->Vc = pp.Vc;
  v->imp = pp.imp;
  v->ctx_sel = pp.ctx_sel;
  v->kept = pp.kept;
  v->energy = pp.energy;
  v->sharp_ids = pp.sharp;
  v->flat_ids = pp.flat;
  v->exact = pp.exact;
  v->exact_bits = pp.bits;
  v->Kp = reinterpret_cast<const uint16_t*>(pp.Kp);
  v->Vp = reinterpret_cast<const uint16_t*>(pp.Vp);
  v->status = pp.status;
  return ISA_OK;
}

isa_status isa_plan(const isa_params* p, const void* q, const void* k, const void* v, void* ws, size_t ws_bytes,
                    void* stream) {
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  if ((s = check_ptr(q, "q", 16)) != ISA_OK || (s = check_ptr(k, "k", 16)) != ISA_OK ||
      (s = check_ptr(v, "v", 16)) != ISA_OK || (s = check_ptr(ws, "workspace", 256)) != ISA_OK)
    return s;
  const PlanLayout L = make_layout(d);
  if (ws_bytes < L.total) return fail(ISA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  if ((s = ensure_init()) != ISA_OK || (s = bind_device_of(q, "q")) != ISA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const PlanPtrs pp = make_ptrs(L, ws);
  cudaError_t e = cudaMemsetAsync(pp.status, 0, 256, st);
  if (e != cudaSuccess) return cuda_fail(e, "status reset");
  e = launch_plan(d, q, k, v, pp, st);
  if (e != cudaSuccess) return cuda_fail(e, "planning launch");
  return ISA_OK;
}

isa_status isa_plan_rope(const isa_params* p, float base, const void* q, const void* k, const void* v, void* q_rot,
                         void* k_rot, void* ws, size_t ws_bytes, void* rope_ws, size_t rope_ws_bytes, void* stream) {
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  if (!(base > 1.f) || !std::isfinite(base)) return fail(ISA_ERR_INVALID_ARG, "base must be finite and > 1");
  if ((s = check_ptr(q, "q", 16)) != ISA_OK || (s = check_ptr(k, "k", 16)) != ISA_OK ||
      (s = check_ptr(v, "v", 16)) != ISA_OK || (s = check_ptr(q_rot, "q_rot", 16)) != ISA_OK ||
      (s = check_ptr(k_rot, "k_rot", 16)) != ISA_OK || (s = check_ptr(ws, "workspace", 256)) != ISA_OK ||
      (s = check_ptr(rope_ws, "rope workspace", 16)) != ISA_OK)
    return s;
  const PlanLayout L = make_layout(d);
  if (ws_bytes < L.total) return fail(ISA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  const size_t need = rope_table_bytes(d);
  if (rope_ws_bytes < need) return fail(ISA_ERR_WORKSPACE, "rope workspace has %zu bytes, needs %zu", rope_ws_bytes, need);
  if ((s = ensure_init()) != ISA_OK || (s = bind_device_of(q, "q")) != ISA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const PlanPtrs pp = make_ptrs(L, ws);
  cudaError_t e = cudaMemsetAsync(pp.status, 0, 256, st);
  if (e != cudaSuccess) return cuda_fail(e, "status reset");
  if ((e = launch_rope_table(d, (double)base, rope_ws, st)) != cudaSuccess) return cuda_fail(e, "rope table launch");
  const RopeArgs ra{static_cast<const float2*>(rope_ws), q_rot, k_rot};
  e = launch_plan(d, q, k, v, pp, st, &ra);
  if (e != cudaSuccess) return cuda_fail(e, "planning launch");
  return ISA_OK;
}

// Sizes, plan pointers and work-list counts of the attention kernels (mode 0:
// ISA items from the plan; mode 1: dense items).
static AttnArgs attn_args(const Dims& d, int mode, const PlanPtrs* pp) {
  const int R = mode == 1 ? 64 : d.b;
  AttnArgs a{};
  a.BH = d.BH;
  a.L = d.L;
  a.L_src = d.L_src;
  a.L_ctx = d.L_ctx;
  a.b = d.b;
  a.T_src = d.T_src;
  a.T_ctx = d.T_ctx;
  a.T_kv = d.T_kv;
  a.T_kv_pad = d.T_kv_pad;
  a.K_sel = d.K_sel;
  a.n_sharp = d.n_sharp;
  a.n_flat = d.n_flat;
  a.n_exact = d.n_exact;
  a.words = d.words;
  a.mode = mode;
  const int G = 128 / R;
  a.items_sharp = (d.n_sharp + G - 1) / G;
  a.items_flat = (d.n_flat + G - 1) / G;
  a.q_tiles = (d.L + 127) / 128;
  a.total_items = mode == 1 ? d.BH * a.q_tiles : d.BH * (a.items_sharp + a.items_flat);
  a.sl2 = d.scale * 1.4426950408889634f;
  if (pp) {
    a.kept = pp->kept;
    a.sharp = pp->sharp;
    a.flat = pp->flat;
    a.exact = pp->exact;
    a.bits = pp->bits;
    a.ctx_sel = pp->ctx_sel;
  }
  a.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  a.inject = g_inject.load(std::memory_order_relaxed);
  return a;
}

static isa_status run_attention(const Dims& d, int mode, const void* q, const void* k, const void* v,
                                const PlanPtrs* pp, void* out, float* lse, int32_t* status, cudaStream_t st) {
  isa_status s;
  const int R = mode == 1 ? 64 : d.b;
  CUtensorMap maps[5];
  const uint64_t rows = (uint64_t)d.BH * d.L;
  if ((s = make_map(&maps[0], q, rows, d.D, R, "q")) != ISA_OK) return s;
  if ((s = make_map(&maps[1], k, rows, d.D, R, "k")) != ISA_OK) return s;
  if ((s = make_map(&maps[2], v, rows, d.D, R, "v")) != ISA_OK) return s;
  if (pp) {
    const uint64_t prow = (uint64_t)d.BH * d.T_kv_pad;
    if ((s = make_map(&maps[3], pp->Kp, prow, d.D, R, "Kp")) != ISA_OK) return s;
    if ((s = make_map(&maps[4], pp->Vp, prow, d.D, R, "Vp")) != ISA_OK) return s;
  } else {
    maps[3] = maps[1];
    maps[4] = maps[2];
  }
  AttnArgs a = attn_args(d, mode, pp);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.status = status;
  if (a.total_items == 0) return ISA_OK;
  const int grid = std::min(sm_count(), a.total_items);
  cudaError_t e = launch_attention(d.D, R, maps, a, grid, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return ISA_OK;
}

// Byte offsets of the backward workspace: lse2 and Delta per row of every
// query block ([BH, T, 2, b] fp32, padded past each block's end), then the
// fp32 gradients of the pooled keys and values.
struct BwdLayout {
  size_t dl, dKc, dVc, total;
};

static BwdLayout bwd_layout(const Dims& d) {
  BwdLayout L{};
  L.dl = 0;
  L.dKc = align256((size_t)d.BH * d.T * d.b * 8);
  L.dVc = L.dKc + align256((size_t)d.BH * d.T_kv_pad * d.D * 4);
  L.total = L.dVc + align256((size_t)d.BH * d.T_kv_pad * d.D * 4);
  return L;
}

isa_status isa_forward(const isa_params* p, const void* q, const void* k, const void* v, const void* ws,
                       size_t ws_bytes, void* out, float* lse, void* stream) {
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  if ((s = check_ptr(q, "q", 16)) != ISA_OK || (s = check_ptr(k, "k", 16)) != ISA_OK ||
      (s = check_ptr(v, "v", 16)) != ISA_OK || (s = check_ptr(ws, "workspace", 256)) != ISA_OK ||
      (s = check_ptr(out, "out", 16)) != ISA_OK)
    return s;
  if (lse && (s = check_ptr(lse, "lse", 4)) != ISA_OK) return s;
  const PlanLayout L = make_layout(d);
  if (ws_bytes < L.total) return fail(ISA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  if ((s = ensure_init()) != ISA_OK || (s = bind_device_of(q, "q")) != ISA_OK) return s;
  const PlanPtrs pp = make_ptrs(L, const_cast<void*>(ws));
  return run_attention(d, 0, q, k, v, &pp, out, lse, pp.status, reinterpret_cast<cudaStream_t>(stream));
}

isa_status isa_dense(const isa_params* p, const void* q, const void* k, const void* v, void* out, float* lse,
                     int32_t* status, void* stream) {
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  if ((s = check_ptr(q, "q", 16)) != ISA_OK || (s = check_ptr(k, "k", 16)) != ISA_OK ||
      (s = check_ptr(v, "v", 16)) != ISA_OK || (s = check_ptr(out, "out", 16)) != ISA_OK)
    return s;
  if (lse && (s = check_ptr(lse, "lse", 4)) != ISA_OK) return s;
  if (status && (s = check_ptr(status, "status", 4)) != ISA_OK) return s;
  if ((s = ensure_init()) != ISA_OK || (s = bind_device_of(q, "q")) != ISA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (status) {
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return cuda_fail(e, "status reset");
  }
  return run_attention(d, 1, q, k, v, nullptr, out, lse, status, st);
}

isa_status isa_backward_workspace_size(const isa_params* p, size_t* bytes) {
  if (!bytes) return fail(ISA_ERR_INVALID_ARG, "bytes is NULL");
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  *bytes = bwd_layout(d).total;
  return ISA_OK;
}

isa_status isa_backward(const isa_params* p, const void* q, const void* k, const void* v, const void* ws,
                        size_t ws_bytes, const void* out, const float* lse, const void* dout, void* dq, void* dk,
                        void* dv, void* bws, size_t bws_bytes, void* stream) {
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  if ((s = check_ptr(q, "q", 16)) != ISA_OK || (s = check_ptr(k, "k", 16)) != ISA_OK ||
      (s = check_ptr(v, "v", 16)) != ISA_OK || (s = check_ptr(ws, "workspace", 256)) != ISA_OK ||
      (s = check_ptr(out, "out", 16)) != ISA_OK || (s = check_ptr(lse, "lse", 4)) != ISA_OK ||
      (s = check_ptr(dout, "dout", 16)) != ISA_OK || (s = check_ptr(dq, "dq", 16)) != ISA_OK ||
      (s = check_ptr(dk, "dk", 16)) != ISA_OK || (s = check_ptr(dv, "dv", 16)) != ISA_OK ||
      (s = check_ptr(bws, "backward workspace", 256)) != ISA_OK)
    return s;
  const PlanLayout L = make_layout(d);
  if (ws_bytes < L.total) return fail(ISA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  const BwdLayout BL = bwd_layout(d);
  if (bws_bytes < BL.total)
    return fail(ISA_ERR_WORKSPACE, "backward workspace has %zu bytes, needs %zu", bws_bytes, BL.total);
  if ((s = ensure_init()) != ISA_OK || (s = bind_device_of(q, "q")) != ISA_OK) return s;
  const PlanPtrs pp = make_ptrs(L, const_cast<void*>(ws));
  CUtensorMap maps[6];
  const uint64_t rows = (uint64_t)d.BH * d.L, prow = (uint64_t)d.BH * d.T_kv_pad;
  if ((s = make_map(&maps[0], q, rows, d.D, d.b, "q")) != ISA_OK) return s;
  if ((s = make_map(&maps[1], k, rows, d.D, d.b, "k")) != ISA_OK) return s;
  if ((s = make_map(&maps[2], v, rows, d.D, d.b, "v")) != ISA_OK) return s;
  if ((s = make_map(&maps[3], pp.Kp, prow, d.D, d.b, "Kp")) != ISA_OK) return s;
  if ((s = make_map(&maps[4], pp.Vp, prow, d.D, d.b, "Vp")) != ISA_OK) return s;
  if ((s = make_map(&maps[5], dout, rows, d.D, d.b, "dout")) != ISA_OK) return s;
  BwdArgs b{};
  b.a = attn_args(d, 0, &pp);
  b.a.status = pp.status;
  b.o = static_cast<const __nv_bfloat16*>(out);
  b.dout = static_cast<const __nv_bfloat16*>(dout);
  b.lse = lse;
  char* w = static_cast<char*>(bws);
  b.dl = reinterpret_cast<float*>(w + BL.dl);
  b.dKc = reinterpret_cast<float*>(w + BL.dKc);
  b.dVc = reinterpret_cast<float*>(w + BL.dVc);
  b.dq = static_cast<__nv_bfloat16*>(dq);
  b.dk = static_cast<__nv_bfloat16*>(dk);
  b.dv = static_cast<__nv_bfloat16*>(dv);
  b.scale = d.scale;
  b.has_pooled = (d.n_flat > 0 && d.n_exact < d.T_kv) ? 1 : 0;
  cudaError_t e = launch_backward(d, maps, b, sm_count(), reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "backward launch");
  return ISA_OK;
}

isa_status isa_coarse_residual(const isa_params* p, float gamma, const void* ws, size_t ws_bytes, void* out,
                               void* stream) {
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  if (!std::isfinite(gamma)) return fail(ISA_ERR_INVALID_ARG, "gamma must be finite");
  if ((s = check_ptr(ws, "workspace", 256)) != ISA_OK || (s = check_ptr(out, "out", 16)) != ISA_OK) return s;
  const PlanLayout L = make_layout(d);
  if (ws_bytes < L.total) return fail(ISA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  if ((s = bind_device_of(out, "out")) != ISA_OK) return s;
  const PlanPtrs pp = make_ptrs(L, const_cast<void*>(ws));
  cudaError_t e = launch_coarse(d, pp, gamma, out, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                                reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "coarse residual launch");
  return ISA_OK;
}

isa_status isa_coarse_residual_backward_workspace_size(const isa_params* p, size_t* bytes) {
  if (!bytes) return fail(ISA_ERR_INVALID_ARG, "bytes is NULL");
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  *bytes = coarse_backward_bytes(d);
  return ISA_OK;
}

isa_status isa_coarse_residual_backward(const isa_params* p, float gamma, const void* ws, size_t ws_bytes,
                                        const void* dout, void* dq, void* dk, void* dv, float* dgamma, void* cws,
                                        size_t cws_bytes, void* stream) {
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  if (!std::isfinite(gamma)) return fail(ISA_ERR_INVALID_ARG, "gamma must be finite");
  if ((s = check_ptr(ws, "workspace", 256)) != ISA_OK || (s = check_ptr(dout, "dout", 16)) != ISA_OK ||
      (s = check_ptr(dq, "dq", 16)) != ISA_OK || (s = check_ptr(dk, "dk", 16)) != ISA_OK ||
      (s = check_ptr(dv, "dv", 16)) != ISA_OK || (s = check_ptr(cws, "coarse workspace", 256)) != ISA_OK)
    return s;
  if (dgamma && (s = check_ptr(dgamma, "dgamma", 4)) != ISA_OK) return s;
  const PlanLayout L = make_layout(d);
  if (ws_bytes < L.total) return fail(ISA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  const size_t need = coarse_backward_bytes(d);
  if (cws_bytes < need) return fail(ISA_ERR_WORKSPACE, "coarse workspace has %zu bytes, needs %zu", cws_bytes, need);
  if ((s = bind_device_of(dq, "dq")) != ISA_OK) return s;
  const PlanPtrs pp = make_ptrs(L, const_cast<void*>(ws));
  cudaError_t e = launch_coarse(d, pp, gamma, nullptr, dout, dq, dk, dv, dgamma, cws,
                                reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "coarse residual backward launch");
  return ISA_OK;
}

isa_status isa_rope_workspace_size(const isa_params* p, size_t* bytes) {
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  if (!bytes) return fail(ISA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = rope_table_bytes(d);
  return ISA_OK;
}

isa_status isa_rope(const isa_params* p, float base, const void* q, const void* k, void* q_out, void* k_out,
                    void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  isa_status s = make_dims(p, &d);
  if (s != ISA_OK) return s;
  if (!(base > 1.f) || !std::isfinite(base)) return fail(ISA_ERR_INVALID_ARG, "base must be finite and > 1");
  if ((s = check_ptr(q, "q", 16)) != ISA_OK || (s = check_ptr(k, "k", 16)) != ISA_OK ||
      (s = check_ptr(q_out, "q_out", 16)) != ISA_OK || (s = check_ptr(k_out, "k_out", 16)) != ISA_OK ||
      (s = check_ptr(ws, "workspace", 16)) != ISA_OK)
    return s;
  const size_t need = rope_table_bytes(d);
  if (ws_bytes < need) return fail(ISA_ERR_WORKSPACE, "rope workspace has %zu bytes, needs %zu", ws_bytes, need);
  if ((s = bind_device_of(q, "q")) != ISA_OK) return s;
  cudaError_t e = launch_rope(d, (double)base, q, k, q_out, k_out, ws, sm_count(), reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rope launch");
  return ISA_OK;
}

const char* isa_last_error(void) { return g_last_error.c_str(); }

const char* isa_version(void) { return "isa-b200 0.1 sm_100a"; }

isa_status isa_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(ns ? ns : kDefaultTimeoutNs, std::memory_order_relaxed);
  return ISA_OK;
}

isa_status isa_set_fault_injection(int32_t mode) {
  if (mode != 0 && mode != 1) return fail(ISA_ERR_INVALID_ARG, "fault injection mode must be 0 or 1");
  g_inject.store(mode, std::memory_order_relaxed);
  return ISA_OK;
}

}  // extern "C"
