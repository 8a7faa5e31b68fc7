// gamma * O_coarse, the low-frequency residual of step (6) of "Method steps
// in detail" (paper.rainbus.top summary card of "LIVEditor-14B: Lightning
// Unified Video Editing via In-Context Sparse Attention"), and its backward.
//
// The card names gamma and O_coarse without defining them.  Reading: O_coarse
// is the output of the block-level pooling attention of its "Block-sparse
// attention and pooling attention" background, computed on the pooled means
// the plan already holds:
//   O_coarse_i = sum_j softmax_j(s Qc_i . Kc_j) Vc_j   over all T blocks,
// added as gamma * O_coarse_i to every token of query block i; gamma is the
// caller's scalar.
//
// The work is T x T x D per head (a few GFLOP at 32K tokens), so these are
// CUDA-core kernels, one CTA per (head, block), 256 threads:
//   coarse_fwd_kernel   scores of block i against all T pooled keys (one warp
//                       per key, float4 lanes), softmax, O_coarse_i, and the
//                       read-modify-write of the block's output rows
//   coarse_bwd_q_kernel per query block i: dO_i = gamma * sum of the block's
//                       dout rows, Delta_i = dO_i . O_i, dS_ij =
//                       P_ij (dO_i . Vc_j - Delta_i), dQc_i = s sum_j dS_ij Kc_j
//                       -> dq rows += dQc_i / n_i; keeps (lse2_i, Delta_i) and
//                       dO_i for the key pass; dgamma partial
//   coarse_bwd_kv_kernel per key block j: dKc_j = s sum_i dS_ij Qc_i,
//                       dVc_j = sum_i P_ij dO_i -> dk, dv rows += (.) / n_j
// Gradients reach the tokens through the pooled means (Kc_j is the mean of
// block j's n_j keys), as in the sparse path's backward.
#include <algorithm>

#include "isa_common.cuh"

namespace isa {
namespace coarse {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
__device__ __forceinline__ float warp_dot(const float* __restrict__ a, const float* __restrict__ b) {
  // D/32 consecutive elements per lane (float4 or float2), reduced over the warp
  const int lane = threadIdx.x & 31;
  float acc = 0.f;
  if constexpr (D == 128) {
    const float4 x = reinterpret_cast<const float4*>(a)[lane], y = reinterpret_cast<const float4*>(b)[lane];
    acc = x.x * y.x + x.y * y.y + x.z * y.z + x.w * y.w;
  } else {
    const float2 x = reinterpret_cast<const float2*>(a)[lane], y = reinterpret_cast<const float2*>(b)[lane];
    acc = x.x * y.x + x.y * y.y;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  return acc;
}

// Block-wide max or sum of one value per thread (all threads must call).
template <bool MAX>
__device__ __forceinline__ float block_reduce(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o = __shfl_xor_sync(0xFFFFFFFFu, v, off);
    v = MAX ? fmaxf(v, o) : v + o;
  }
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < kWarps; ++w) r = MAX ? fmaxf(r, red[w]) : r + red[w];
  return r;
}

// Row i of P = softmax(s Qc Kc^T) into pr[0..T) (shared), its log2 normaliser
// returned: scores in log2 units, one warp per key block.
template <int D>
__device__ float coarse_row(const float* __restrict__ Qc_i, const float* __restrict__ Kc, int T, float sl2,
                            float* pr, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int j = warp; j < T; j += kWarps) {
    const float d = warp_dot<D>(Qc_i, Kc + (size_t)j * D);
    if (lane == 0) pr[j] = d * sl2;
  }
  __syncthreads();
  float m = -INFINITY;
  for (int j = threadIdx.x; j < T; j += kThreads) m = fmaxf(m, pr[j]);
  m = block_reduce<true>(m, red);
  float l = 0.f;
  for (int j = threadIdx.x; j < T; j += kThreads) {
    const float e = exp2f(pr[j] - m);
    pr[j] = e;
    l += e;
  }
  l = block_reduce<false>(l, red);
  const float inv = 1.f / l;
  for (int j = threadIdx.x; j < T; j += kThreads) pr[j] *= inv;
  __syncthreads();
  return m + __log2f(l);
}

// oc[0..D) = sum_j pr[j] Vc_j (shared), two halves of the threads over j.
template <int D>
__device__ void coarse_combine(const float* pr, const float* __restrict__ Vc, int T, float* oc, float* part) {
  constexpr int SPLIT = kThreads / D;   // 2 (D=128) or 4 (D=64) partial sums per column
  const int d = threadIdx.x % D, h = threadIdx.x / D;
  float acc = 0.f;
  for (int j = h; j < T; j += SPLIT) acc = fmaf(pr[j], Vc[(size_t)j * D + d], acc);
  part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
    for (int k = 0; k < SPLIT; ++k) s += part[k * D + threadIdx.x];
    oc[threadIdx.x] = s;
  }
  __syncthreads();
}

// rows [t0, t0+n) of x (bf16 [.., D]) += scale * v (shared fp32 [D])
template <int D>
__device__ void add_rows(__nv_bfloat16* x, size_t t0, int n, const float* v, float scale) {
  for (int e = threadIdx.x; e < n * (D / 8); e += kThreads) {
    const int r = e / (D / 8), c = (e % (D / 8)) * 8;
    uint4* p = reinterpret_cast<uint4*>(x + (t0 + r) * D + c);
    uint4 w = *p;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(h[k]);
      h[k] = __floats2bfloat162_rn(fmaf(scale, v[c + 2 * k], f.x), fmaf(scale, v[c + 2 * k + 1], f.y));
    }
    *p = w;
  }
}

struct CoarseArgs {
  const float *Qc, *Kc, *Vc;   // plan: [BH, T, D]
  int T, T_src, L, L_src, L_ctx, b;
  float sl2, scale, gamma;
  __nv_bfloat16* out;          // forward: out += gamma * O_coarse
  const __nv_bfloat16* dout;   // backward
  __nv_bfloat16 *dq, *dk, *dv;
  float* dgamma;               // [BH] or null
  float2* stat;                // [BH, T] (lse2_i, Delta_i)
  float* dO;                   // [BH, T, D] gamma * block sums of dout
};

template <int D>
__global__ void __launch_bounds__(kThreads) coarse_fwd_kernel(const CoarseArgs a) {
  extern __shared__ __align__(16) float sm[];
  float* oc = sm;                  // D
  float* part = oc + D;            // kThreads
  float* red = part + kThreads;    // kWarps
  float* pr = red + kWarps;        // T
  const int bh = blockIdx.x, i = blockIdx.y;
  const size_t hb = (size_t)bh * a.T * D;
  coarse_row<D>(a.Qc + hb + (size_t)i * D, a.Kc + hb, a.T, a.sl2, pr, red);
  coarse_combine<D>(pr, a.Vc + hb, a.T, oc, part);
  const int2 sp = block_span(i, a.L_src, a.L_ctx, a.b, a.T_src);
  add_rows<D>(a.out, (size_t)bh * a.L + sp.x, sp.y, oc, a.gamma);
}

template <int D>
__global__ void __launch_bounds__(kThreads) coarse_bwd_q_kernel(const CoarseArgs a) {
  // D-sized arrays first: dO is read as float4 / float2 by warp_dot
  extern __shared__ __align__(16) float sm[];
  float* oc = sm;                  // D: O_i
  float* dO = oc + D;              // D: gamma * sum of dout rows
  float* dq = dO + D;              // D
  float* part = dq + D;            // kThreads
  float* red = part + kThreads;    // kWarps
  float* pr = red + kWarps;        // T: P_ij, then dS_ij
  const int bh = blockIdx.x, i = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t hb = (size_t)bh * a.T * D;
  const float lse2 = coarse_row<D>(a.Qc + hb + (size_t)i * D, a.Kc + hb, a.T, a.sl2, pr, red);
  coarse_combine<D>(pr, a.Vc + hb, a.T, oc, part);
  // sum of the block's dout rows, one column per thread (split over rows)
  const int2 sp = block_span(i, a.L_src, a.L_ctx, a.b, a.T_src);
  {
    constexpr int SPLIT = kThreads / D;
    const int d = threadIdx.x % D, h = threadIdx.x / D;
    float acc = 0.f;
    for (int r = h; r < sp.y; r += SPLIT) acc += __bfloat162float(a.dout[((size_t)bh * a.L + sp.x + r) * D + d]);
    part[threadIdx.x] = acc;
    __syncthreads();
    if (threadIdx.x < D) {
      float s = 0.f;
      for (int k = 0; k < SPLIT; ++k) s += part[k * D + threadIdx.x];
      dO[threadIdx.x] = s;
    }
    __syncthreads();
  }
  // dgamma partial = (sum of dout rows) . O_i; then dO *= gamma; Delta = dO . O_i
  float g = threadIdx.x < D ? dO[threadIdx.x] * oc[threadIdx.x] : 0.f;
  g = block_reduce<false>(g, red);
  if (threadIdx.x == 0 && a.dgamma) atomicAdd(a.dgamma + bh, g);
  if (threadIdx.x < D) dO[threadIdx.x] *= a.gamma;
  __syncthreads();
  const float delta = a.gamma * g;
  if (threadIdx.x == 0) a.stat[(size_t)bh * a.T + i] = make_float2(lse2, delta);
  if (threadIdx.x < D) a.dO[hb + (size_t)i * D + threadIdx.x] = dO[threadIdx.x];
  // dS_ij = P_ij (dO . Vc_j - Delta), in place of P_ij
  for (int j = warp; j < a.T; j += kWarps) {
    const float dp = warp_dot<D>(dO, a.Vc + hb + (size_t)j * D);
    if (lane == 0) pr[j] = pr[j] * (dp - delta);
  }
  __syncthreads();
  // dQc_i = s sum_j dS_ij Kc_j
  coarse_combine<D>(pr, a.Kc + hb, a.T, dq, part);
  add_rows<D>(a.dq, (size_t)bh * a.L + sp.x, sp.y, dq, a.scale / (float)sp.y);
}

template <int D>
__global__ void __launch_bounds__(kThreads) coarse_bwd_kv_kernel(const CoarseArgs a) {
  // D-sized arrays first: kc and vc are read as float4 / float2 by warp_dot
  extern __shared__ __align__(16) float sm[];
  float* kc = sm;                  // D: Kc_j
  float* vc = kc + D;              // D: Vc_j
  float* gk = vc + D;              // D
  float* gv = gk + D;              // D
  float* part = gv + D;            // kThreads
  float* pj = part + kThreads;     // T: P_ij over query blocks i
  float* sj = pj + a.T;            // T: dS_ij
  const int bh = blockIdx.x, j = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t hb = (size_t)bh * a.T * D;
  if (threadIdx.x < D) {
    kc[threadIdx.x] = a.Kc[hb + (size_t)j * D + threadIdx.x];
    vc[threadIdx.x] = a.Vc[hb + (size_t)j * D + threadIdx.x];
  }
  __syncthreads();
  for (int i = warp; i < a.T; i += kWarps) {
    const float s = warp_dot<D>(a.Qc + hb + (size_t)i * D, kc);
    const float dp = warp_dot<D>(a.dO + hb + (size_t)i * D, vc);
    if (lane == 0) {
      const float2 st = a.stat[(size_t)bh * a.T + i];
      const float p = exp2f(s * a.sl2 - st.x);
      pj[i] = p;
      sj[i] = p * (dp - st.y);
    }
  }
  __syncthreads();
  // dKc_j = s sum_i dS_ij Qc_i, dVc_j = sum_i P_ij dO_i
  coarse_combine<D>(sj, a.Qc + hb, a.T, gk, part);
  coarse_combine<D>(pj, a.dO + hb, a.T, gv, part);
  const int2 sp = block_span(j, a.L_src, a.L_ctx, a.b, a.T_src);
  add_rows<D>(a.dk, (size_t)bh * a.L + sp.x, sp.y, gk, a.scale / (float)sp.y);
  add_rows<D>(a.dv, (size_t)bh * a.L + sp.x, sp.y, gv, 1.f / (float)sp.y);
}

template <int D>
static cudaError_t launch_t(const Dims& d, const CoarseArgs& a, bool backward, cudaStream_t st) {
  const dim3 grid(d.BH, d.T);
  if (!backward) {
    const size_t sm = (size_t)(d.T + D + kThreads + kWarps) * 4;
    static bool attr = false;
    if (!attr) {
      cudaError_t e = cudaFuncSetAttribute(coarse_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
      if (e != cudaSuccess) return e;
      attr = true;
    }
    coarse_fwd_kernel<D><<<grid, kThreads, sm, st>>>(a);
    return cudaGetLastError();
  }
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(coarse_bwd_q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, 80 * 1024);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(coarse_bwd_kv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, 80 * 1024);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const size_t smq = (size_t)(d.T + 3 * D + kThreads + kWarps) * 4;
  coarse_bwd_q_kernel<D><<<grid, kThreads, smq, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smk = (size_t)(4 * D + 2 * d.T + kThreads) * 4;
  coarse_bwd_kv_kernel<D><<<grid, kThreads, smk, st>>>(a);
  return cudaGetLastError();
}

}  // namespace coarse

size_t coarse_backward_bytes(const Dims& d) {
  const size_t stat = ((size_t)d.BH * d.T * 8 + 255) & ~(size_t)255;
  return stat + (size_t)d.BH * d.T * d.D * 4;
}

cudaError_t launch_coarse(const Dims& d, const PlanPtrs& pp, float gamma, void* out, const void* dout, void* dq,
                          void* dk, void* dv, float* dgamma, void* cws, cudaStream_t st) {
  coarse::CoarseArgs a{};
  a.Qc = pp.Qc;
  a.Kc = pp.Kc;
  a.Vc = pp.Vc;
  a.T = d.T;
  a.T_src = d.T_src;
  a.L = d.L;
  a.L_src = d.L_src;
  a.L_ctx = d.L_ctx;
  a.b = d.b;
  a.scale = d.scale;
  a.sl2 = d.scale * coarse::kLog2e;
  a.gamma = gamma;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.dout = static_cast<const __nv_bfloat16*>(dout);
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.dgamma = dgamma;
  const bool backward = dout != nullptr;
  if (backward) {
    char* w = static_cast<char*>(cws);
    a.stat = reinterpret_cast<float2*>(w);
    a.dO = reinterpret_cast<float*>(w + (((size_t)d.BH * d.T * 8 + 255) & ~(size_t)255));
    if (dgamma) {
      cudaError_t e = cudaMemsetAsync(dgamma, 0, (size_t)d.BH * sizeof(float), st);
      if (e != cudaSuccess) return e;
    }
  }
  if (d.D == 128) return coarse::launch_t<128>(d, a, backward, st);
  if (d.D == 64) return coarse::launch_t<64>(d, a, backward, st);
  return cudaErrorInvalidValue;
}

}  // namespace isa
