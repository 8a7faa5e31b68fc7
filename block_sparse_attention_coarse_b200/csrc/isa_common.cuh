// Shared definitions of the ISA CUDA library: plan-workspace layout and the
// sm_100a device primitives (mbarrier with bounded waits, TMA tile loads,
// tcgen05 MMA / TMEM access) written as inline PTX.
#pragma once

#include <atomic>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/isa.h"

namespace isa {

// ---------------------------------------------------------------------------
// problem sizes derived from isa_params (host and device)
// ---------------------------------------------------------------------------

struct Dims {
  int B, H, BH, D, L_src, L_ctx, L, b;
  int T_src, T_ctx, T, K_sel, T_kv, n_flat, n_sharp, n_exact, T_kv_pad, words;
  float scale;
};

// Byte offsets of every plan array inside the caller's workspace.
struct PlanLayout {
  size_t status, Qc, Kc, Vc, imp, ctx_sel, kept, energy, sharp, flat, exact, bits, Kp, Vp, total;
};

struct PlanPtrs {
  int* status;
  float *Qc, *Kc, *Vc, *imp, *energy;
  int *ctx_sel, *kept, *sharp, *flat, *exact;
  uint32_t* bits;
  __nv_bfloat16 *Kp, *Vp;
};

// Argument block of the attention kernel (isa_attn.cu).
struct AttnArgs {
  int BH, L, L_src, L_ctx, b, T_src, T_ctx, T_kv, T_kv_pad, K_sel, n_sharp, n_flat, n_exact, words;
  int mode;                  // 0 = ISA sparse, 1 = dense
  int items_sharp, items_flat, q_tiles, total_items;
  float sl2;                 // softmax scale * log2(e)
  const int* kept;
  const int* sharp;
  const int* flat;
  const int* exact;
  const uint32_t* bits;
  const int* ctx_sel;
  __nv_bfloat16* out;
  float* lse;
  int* status;
  unsigned long long timeout_ns;
  int inject;
};

// Argument block of the backward kernels (isa_bwd.cu).  `a` carries the
// plan, the sizes and the forward's sparse work list (mode 0).
struct BwdArgs {
  AttnArgs a;
  const __nv_bfloat16* o;      // forward output [BH*L, D]
  const __nv_bfloat16* dout;   // gradient of the output [BH*L, D]
  const float* lse;            // forward natural-log normalisers [BH*L]
  float* dl;                   // [BH, T, 2, b]: per block, the rows' lse * log2 e, then their rowsum(dout * o);
                               // (inf, 0) past a block's end
  float* dKc;                  // [BH, T_kv_pad, D] gradient of the pooled keys (scaled)
  float* dVc;                  // [BH, T_kv_pad, D] gradient of the pooled values
  __nv_bfloat16 *dq, *dk, *dv; // [BH*L, D]
  float scale;                 // softmax scale s
  int has_pooled;              // some flat block has pooled columns (dKc/dVc are filled)
  int kv_pooled;               // key/value-stationary launch over pooled rows (1) or kept blocks (0)
  int kv_tiles;                // key/value tiles per head of that launch
  int kv_total;                // BH * kv_tiles
};

// Decoupled RoPE folded into the pooling pass (isa_plan_rope): the (cos, sin)
// table and where the rotated Q and K rows go.
struct RopeArgs {
  const float2* tab;   // [max(L_src, L_ctx), D/2] (cos, sin) per segment position and pair
  void* q_rot;         // bf16 [BH*L, D]; may be q (in place)
  void* k_rot;         // bf16 [BH*L, D]; may be k (in place)
};

// launchers (host)
cudaError_t launch_plan(const Dims& dm, const void* q, const void* k, const void* v, const PlanPtrs& pp,
                        cudaStream_t st, const RopeArgs* rope = nullptr);
cudaError_t launch_attention(int D, int R, const CUtensorMap* maps, const AttnArgs& a, int grid, cudaStream_t st);
cudaError_t launch_backward(const Dims& d, const CUtensorMap* maps, BwdArgs& b, int sm_count, cudaStream_t st);
size_t coarse_backward_bytes(const Dims& d);
cudaError_t launch_coarse(const Dims& d, const PlanPtrs& pp, float gamma, void* out, const void* dout, void* dq,
                          void* dk, void* dv, float* dgamma, void* cws, cudaStream_t st);
size_t rope_table_bytes(const Dims& d);
cudaError_t launch_rope(const Dims& d, double base, const void* q, const void* k, void* qo, void* ko, void* tab,
                        int sm_count, cudaStream_t st);
cudaError_t launch_rope_table(const Dims& d, double base, void* tab, cudaStream_t st);
void set_last_error(const char* msg);
isa_status bind_device_of(const void* ptr, const char* name);

// Kernel attributes (the dynamic shared-memory limit) belong to the module
// loaded on each device, so they are set on the first launch on every
// device, not once per process.  `done` holds one bit per device 0..63;
// devices beyond that set the attributes on every launch.
template <class F>
cudaError_t once_per_device(std::atomic<unsigned long long>& done, F&& set) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = set();
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

constexpr int kMaxT = 8192;      // blocks per head
constexpr int kMaxTkv = 6144;    // kept blocks per head
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------
#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// -- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of phase `parity` of `bar` (never suspends the thread).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Shared state of the bounded waits of one CTA.
struct WaitCtl {
  volatile int* abort;       // shared-memory flag: some wait of this CTA ran out
  int* status;               // device status word (may be null)
  uint64_t limit_ns;
};

// Waits for the phase `parity` of `bar`.  Gives up when the CTA's abort flag
// is raised or, after limit_ns, raises it and records the timeout.  Returns
// true when the phase completed.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort) return false;
    if (globaltimer() - t0 > w.limit_ns) {
      *w.abort = 1;
      if (w.status) atomicExch(w.status, (int)ISA_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

// Same, but ignores the abort flag: used on the way out to let copies that
// are already in flight land before the CTA exits.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit_ns) return false;
  }
  return true;
}

// -- TMA ----------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
// 2-D tiled load of box (x = column, y = row) into shared memory, completing
// on `bar` with a byte count.  No multicast.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 1-D bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned)
// from global to shared memory, completing on `bar` with a byte count.  No
// multicast.
__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// -- tcgen05 ------------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Whole warp.  Writes the TMEM base address to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Arrive on `bar` once every tcgen05.mma issued so far by this thread completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem], A read from tensor memory.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same three ops for a whole converged warp: one lane, picked by
// elect.sync, issues the instruction.  Called with warp-uniform operands, so
// the descriptors stay in uniform registers and no lane-by-lane loop is
// needed to issue them.
__device__ __forceinline__ void mma_ss_elect(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit_elect(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

#define ISA_R32(a) \
  "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]), "=r"(a[8]),     \
      "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]), "=r"(a[16]),        \
      "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), "=r"(a[24]),       \
      "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31])
#define ISA_W32(a) \
  "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]), "r"(a[8]), "r"(a[9]),      \
      "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]), "r"(a[15]), "r"(a[16]), "r"(a[17]), "r"(a[18]),   \
      "r"(a[19]), "r"(a[20]), "r"(a[21]), "r"(a[22]), "r"(a[23]), "r"(a[24]), "r"(a[25]), "r"(a[26]), "r"(a[27]),   \
      "r"(a[28]), "r"(a[29]), "r"(a[30]), "r"(a[31])

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%"
      "18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      ISA_W32(r)
      : "memory");
}
#define ISA_W16(a) \
  "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]), "r"(a[8]), "r"(a[9]),      \
      "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]), "r"(a[15])
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      ISA_W16(r)
      : "memory");
}
#define ISA_R16(a) \
  "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]), "=r"(a[8]),     \
      "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15])
// TMEM loads that end in their own tcgen05.wait::ld, all in one asm
// statement: the compiler sees the destination registers only once the
// data has landed, so no instruction (a spill included) can read one early.
// Two 32x32b.x16 groups (16 columns of lane base+i for thread i, each).
__device__ __forceinline__ void tmem_ld16_pair_sync(uint32_t ta, uint32_t (&ra)[16], uint32_t tb,
                                                    uint32_t (&rb)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31},"
      " [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ISA_R16(ra), ISA_R16(rb)
      : "r"(ta), "r"(tb)
      : "memory");
}
// One 32x32b.x16 group and the wait.
__device__ __forceinline__ void tmem_ld16_sync(uint32_t ta, uint32_t (&ra)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ISA_R16(ra)
      : "r"(ta)
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of an operand stored with the 128-byte
// swizzle that TMA's SWIZZLE_128B writes: rows of 128 bytes, 8-row groups of
// 1024 bytes.  lbo/sbo in bytes.  Bits: [0,14) start>>4, [16,30) lbo>>4,
// [32,46) sbo>>4, [46,48) version 1, [61,64) layout 2 (128B swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B,
// A K-major, B K-major (b_mn = 0) or MN-major (b_mn = 1), M x N tile.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int b_mn) {
  return (1u << 4)                       // D format f32
         | (1u << 7)                     // A format bf16
         | (1u << 10)                    // B format bf16
         | ((uint32_t)b_mn << 16)        // B major
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 3-input maximum (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// Packed fp32 pair arithmetic (one sm_100 instruction for two values).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Order-preserving map of a float to an unsigned key.
__device__ __forceinline__ uint32_t f2ord(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The k-th largest of key[0..n) as an order key (f2ord), 1 <= k <= n, by one
// warp: a radix select over the order keys, 8 bits per pass from the top,
// with a 256-bin histogram per pass in `hist` (shared memory, 256 words,
// this warp's alone).  Each pass counts the keys that match the digits
// chosen so far; the lanes scan the bins from the top digit down (lane l
// holds bins 255-8l .. 248-8l) and keep the digit at which the running count
// reaches the remaining rank.
__device__ inline uint32_t warp_kth_largest(const float* key, int n, int k, uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, pmask = 0;
  uint32_t kk = (uint32_t)k;   // rank of the wanted key among those matching prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0u;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const uint32_t o = f2ord(key[i]);
      if ((o & pmask) == prefix) atomicAdd(&hist[(o >> shift) & 255u], 1u);
    }
    __syncwarp();
    uint32_t c[8], sum = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      c[j] = hist[255 - 8 * lane - j];
      sum += c[j];
    }
    uint32_t incl = sum;   // keys in the bins of lanes 0..lane (digits from the top)
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += v;
    }
    const uint32_t excl = incl - sum;
    const int src = __ffs(__ballot_sync(0xFFFFFFFFu, excl < kk && kk <= incl)) - 1;
    int d = 0;
    uint32_t above = 0u;
    if (lane == src) {
      uint32_t run = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (run + c[j] >= kk) {
          d = 255 - 8 * lane - j;
          above = run;
          break;
        }
        run += c[j];
      }
    }
    d = __shfl_sync(0xFFFFFFFFu, d, src);
    above = __shfl_sync(0xFFFFFFFFu, above, src);
    prefix |= (uint32_t)d << shift;
    pmask |= 255u << shift;
    kk -= above;
    __syncwarp();   // every lane has read the bins before the next pass clears them
  }
  return prefix;
}

// One warp selects the k largest of key[0..n) (shared memory), ties to the
// lower index, writing the chosen indices in ascending order to out[0..k)
// and, when bits != nullptr, the selection as a bitmap of ceil(n/32) words.
// hist: 256 words of shared memory for this warp alone.
__device__ inline void warp_topk(const float* key, int n, int k, int* out, uint32_t* bits, uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  if (k >= n) {
    for (int i = lane; i < n; i += 32) out[i] = i;
    if (bits)
      for (int w = lane; w < (n + 31) / 32; w += 32) {
        int rem = n - w * 32;
        bits[w] = rem >= 32 ? 0xFFFFFFFFu : ((1u << rem) - 1u);
      }
    return;
  }
  // t: the k-th largest order key (0 when k == 0: nothing is selected)
  const uint32_t t = k > 0 ? warp_kth_largest(key, n, k, hist) : 0u;
  int gt = 0;
  if (k > 0) {
#pragma unroll 4
    for (int i = lane; i < n; i += 32) gt += f2ord(key[i]) > t;
    gt = __reduce_add_sync(0xFFFFFFFFu, gt);
  }
  const int need_eq = k - gt;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base = 0, eq_seen = 0;
  for (int i0 = 0; i0 < n; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t o = i < n ? f2ord(key[i]) : 0u;
    const bool valid = (i < n) && (k > 0);
    const bool is_gt = valid && o > t;
    const bool is_eq = valid && o == t;
    const uint32_t eqm = __ballot_sync(0xFFFFFFFFu, is_eq);
    const int eq_rank = eq_seen + __popc(eqm & lt_mask);
    const bool sel = is_gt || (is_eq && eq_rank < need_eq);
    const uint32_t selm = __ballot_sync(0xFFFFFFFFu, sel);
    if (sel) out[base + __popc(selm & lt_mask)] = i;
    if (bits && lane == 0) bits[i0 >> 5] = selm;
    base += __popc(selm);
    eq_seen += __popc(eqm);
  }
}

// One RoPE pair (2i, 2i+1) of bf16 values rotated by the angle whose
// (cos, sin) is cs, in fp32, rounded once to bf16 (nearest even).  The
// standalone rotation and the pooling pass share it, so both give the same
// bits.
__device__ __forceinline__ uint32_t rot_pair(uint32_t xv, float2 cs) {
  const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&xv);
  const float x0 = __low2float(x), x1 = __high2float(x);
  const float y0 = fmaf(x0, cs.x, -x1 * cs.y);
  const float y1 = fmaf(x0, cs.y, x1 * cs.x);
  const __nv_bfloat162 y = __floats2bfloat162_rn(y0, y1);
  return *reinterpret_cast<const uint32_t*>(&y);
}

// Token span of block `id` (source blocks first, each segment blocked on its own).
__device__ __forceinline__ int2 block_span(int id, int L_src, int L_ctx, int b, int T_src) {
  if (id < T_src) {
    const int s = id * b;
    return make_int2(s, min(b, L_src - s));
  }
  const int s = (id - T_src) * b;
  return make_int2(L_src + s, min(b, L_ctx - s));
}

#endif  // __CUDACC__

}  // namespace isa
