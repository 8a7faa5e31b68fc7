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
//   coarse_fwd_kernel   scores of up to 8 query blocks against all T pooled keys
//                       (one key per thread), softmax, O_coarse, and the
//                       read-modify-write of the blocks' output rows
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
constexpr float kLog2e = 1.4426950408889634f;

constexpr int kRows = 8;           // most query (key) blocks per CTA

// Softmax of rows r < nr of pr[r * ld .. + T) in place (log2-unit scores),
// one warp per row; lse2[r] receives each row's log2 normaliser.
__device__ void rows_softmax(float* pr, int ld, int T, int nr, float* lse2) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp < nr) {
    float* row = pr + (size_t)warp * ld;
    float m = -INFINITY;
    for (int j = lane; j < T; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    float l = 0.f;
    for (int j = lane; j < T; j += 32) {
      const float e = exp2f(row[j] - m);
      row[j] = e;
      l += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
    const float inv = 1.f / l;
    for (int j = lane; j < T; j += 32) row[j] *= inv;
    if (lane == 0) lse2[warp] = m + __log2f(l);
  }
  __syncthreads();
}

// out[r][d] = sum_j w[r * ld + j] X[j][d] for r < nr (shared out [kRows][D]):
// each thread owns one column and a contiguous slice of j, with kRows
// accumulators, so every X row is read once for all nr rows, and the
// weights of 4 consecutive j come in one 16-byte broadcast load (ld is a
// multiple of 4 and w is zero in [T, ld)); slices combined through `part`.
template <int D>
__device__ void rows_combine(const float* w, int ld, int nr, const float* __restrict__ X, int T, float* out,
                             float* part) {
  constexpr int SPLIT = kThreads / D;
  const int d = threadIdx.x % D, h = threadIdx.x / D;
  const int chunk = ((ld / 4 + SPLIT - 1) / SPLIT) * 4;
  const int j0 = h * chunk, j1 = min(j0 + chunk, ld);
  float acc[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) acc[r] = 0.f;
  for (int j = j0; j < j1; j += 4) {
    float x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = (j + i < T) ? X[(size_t)(j + i) * D + d] : 0.f;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      if (r < nr) {
        const float4 wv = *reinterpret_cast<const float4*>(w + (size_t)r * ld + j);
        acc[r] = fmaf(wv.x, x[0], fmaf(wv.y, x[1], fmaf(wv.z, x[2], fmaf(wv.w, x[3], acc[r]))));
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRows; ++r) part[(h * kRows + r) * D + d] = acc[r];
  __syncthreads();
  for (int e = threadIdx.x; e < nr * D; e += kThreads) {
    const int r = e / D, c = e % D;
    float sum = 0.f;
    for (int k = 0; k < SPLIT; ++k) sum += part[(k * kRows + r) * D + c];
    out[r * D + c] = sum;
  }
  __syncthreads();
}

// acc[r] = A[r] . x for r < nr: the rows of A in shared memory (read as
// 16-byte broadcasts: every lane of a warp reads the same address), x one
// row of global memory per thread.  Threads take different x rows, so no
// shuffle reduction is needed.
template <int D>
__device__ __forceinline__ void row_dots(const float* A, int nr, const float* __restrict__ x, float (&acc)[kRows]) {
#pragma unroll
  for (int r = 0; r < kRows; ++r) acc[r] = 0.f;
#pragma unroll 4
  for (int c = 0; c < D; c += 4) {
    const float4 xv = *reinterpret_cast<const float4*>(x + c);
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      if (r < nr) {
        const float4 av = *reinterpret_cast<const float4*>(A + r * D + c);
        acc[r] = fmaf(av.x, xv.x, fmaf(av.y, xv.y, fmaf(av.z, xv.z, fmaf(av.w, xv.w, acc[r]))));
      }
    }
  }
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
  int rows;                    // query (key) blocks per CTA, <= kRows
  float sl2, scale, gamma;
  __nv_bfloat16* out;          // forward: out += gamma * O_coarse
  const __nv_bfloat16* dout;   // backward
  __nv_bfloat16 *dq, *dk, *dv;
  float* dgamma;               // [BH] or null
  float2* stat;                // [BH, T] (lse2_i, Delta_i)
  float* dO;                   // [BH, T, D] gamma * block sums of dout
};

// Shared memory: D-vectors first (read as float4 / float2), then the
// combine scratch, then the [rows][T] score rows.
template <int D>
constexpr int kVecFloats = 2 * kRows * D;
template <int D>
constexpr int kPartFloats = (kThreads / D) * kRows * D;

template <int D>
__global__ void __launch_bounds__(kThreads) coarse_fwd_kernel(const CoarseArgs a) {
  extern __shared__ __align__(16) float sm[];
  float* qs = sm;                          // [kRows][D] Qc rows
  float* oc = qs + kRows * D;              // [kRows][D] O_coarse rows
  float* part = oc + kRows * D;            // combine scratch
  float* lse2 = part + kPartFloats<D>;     // [kRows]
  float* pr = lse2 + kRows;                // [rows][ld], zero past T
  const int bh = blockIdx.x, i0 = blockIdx.y * a.rows;
  const int nr = min(a.rows, a.T - i0);
  const int ld = (a.T + 3) & ~3;
  const size_t hb = (size_t)bh * a.T * D;
  for (int e = threadIdx.x; e < nr * D; e += kThreads) qs[e] = a.Qc[hb + (size_t)i0 * D + e];
  __syncthreads();
  // scores: one key block per thread, against all nr query rows
  for (int j = threadIdx.x; j < ld; j += kThreads) {
    float acc[kRows];
    if (j < a.T) row_dots<D>(qs, nr, a.Kc + hb + (size_t)j * D, acc);
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      if (r < nr) pr[(size_t)r * ld + j] = j < a.T ? acc[r] * a.sl2 : 0.f;
  }
  __syncthreads();
  rows_softmax(pr, ld, a.T, nr, lse2);
  rows_combine<D>(pr, ld, nr, a.Vc + hb, a.T, oc, part);
  for (int r = 0; r < nr; ++r) {
    const int2 sp = block_span(i0 + r, a.L_src, a.L_ctx, a.b, a.T_src);
    add_rows<D>(a.out, (size_t)bh * a.L + sp.x, sp.y, oc + r * D, a.gamma);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) coarse_bwd_q_kernel(const CoarseArgs a) {
  extern __shared__ __align__(16) float sm[];
  float* dO = sm;                          // [kRows][D] gamma * dout block sums (read as fragments)
  float* oc = dO + kRows * D;              // [kRows][D] O_coarse rows, then dQc rows
  float* part = oc + kRows * D;            // combine scratch
  float* lse2 = part + kPartFloats<D>;     // [kRows]
  float* pr = lse2 + kRows;                // [rows][ld] P, then dS; zero past T
  const int bh = blockIdx.x, i0 = blockIdx.y * a.rows;
  const int nr = min(a.rows, a.T - i0);
  const int ld = (a.T + 3) & ~3;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t hb = (size_t)bh * a.T * D;
  // scores and softmax, as in the forward (Qc rows staged in dO's space)
  for (int e = threadIdx.x; e < nr * D; e += kThreads) dO[e] = a.Qc[hb + (size_t)i0 * D + e];
  __syncthreads();
  for (int j = threadIdx.x; j < ld; j += kThreads) {
    float acc[kRows];
    if (j < a.T) row_dots<D>(dO, nr, a.Kc + hb + (size_t)j * D, acc);
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      if (r < nr) pr[(size_t)r * ld + j] = j < a.T ? acc[r] * a.sl2 : 0.f;
  }
  __syncthreads();
  rows_softmax(pr, ld, a.T, nr, lse2);
  rows_combine<D>(pr, ld, nr, a.Vc + hb, a.T, oc, part);
  // block sums of dout: thread = column, rows of block i0+r split over the thread slices
  {
    constexpr int SPLIT = kThreads / D;
    const int d = threadIdx.x % D, h = threadIdx.x / D;
    for (int r = 0; r < nr; ++r) {
      const int2 sp = block_span(i0 + r, a.L_src, a.L_ctx, a.b, a.T_src);
      float acc = 0.f;
      for (int t = h; t < sp.y; t += SPLIT) acc += __bfloat162float(a.dout[((size_t)bh * a.L + sp.x + t) * D + d]);
      part[(h * kRows + r) * D + d] = acc;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < nr * D; e += kThreads) {
      const int r = e / D, c = e % D;
      float sum = 0.f;
      for (int k = 0; k < SPLIT; ++k) sum += part[(k * kRows + r) * D + c];
      dO[e] = sum;
    }
    __syncthreads();
  }
  // per row: g = (dout sum) . O (dgamma), then dO *= gamma, Delta = gamma g;
  // one warp per row
  if (warp < nr) {
    float g = 0.f;
    for (int c = lane; c < D; c += 32) g = fmaf(dO[warp * D + c], oc[warp * D + c], g);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) g += __shfl_xor_sync(0xFFFFFFFFu, g, off);
    for (int c = lane; c < D; c += 32) {
      const float x = a.gamma * dO[warp * D + c];
      dO[warp * D + c] = x;
      a.dO[hb + (size_t)(i0 + warp) * D + c] = x;
    }
    if (lane == 0) {
      a.stat[(size_t)bh * a.T + i0 + warp] = make_float2(lse2[warp], a.gamma * g);
      if (a.dgamma) atomicAdd(a.dgamma + bh, g);
      lse2[warp] = a.gamma * g;   // Delta of the row, for the dS pass
    }
  }
  __syncthreads();
  // dS_rj = P_rj (dO_r . Vc_j - Delta_r), in place; one key block per thread
  for (int j = threadIdx.x; j < a.T; j += kThreads) {
    float dp[kRows];
    row_dots<D>(dO, nr, a.Vc + hb + (size_t)j * D, dp);
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      if (r < nr) pr[(size_t)r * ld + j] *= dp[r] - lse2[r];
  }
  __syncthreads();
  // dQc_r = s sum_j dS_rj Kc_j  -> dq rows of block i0+r += dQc_r / n
  rows_combine<D>(pr, ld, nr, a.Kc + hb, a.T, oc, part);
  for (int r = 0; r < nr; ++r) {
    const int2 sp = block_span(i0 + r, a.L_src, a.L_ctx, a.b, a.T_src);
    add_rows<D>(a.dq, (size_t)bh * a.L + sp.x, sp.y, oc + r * D, a.scale / (float)sp.y);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) coarse_bwd_kv_kernel(const CoarseArgs a) {
  extern __shared__ __align__(16) float sm[];
  float* kc = sm;                          // [kRows][D] Kc rows, then dKc rows
  float* vc = kc + kRows * D;              // [kRows][D] Vc rows, then dVc rows
  float* part = vc + kRows * D;            // combine scratch
  const int ld = (a.T + 3) & ~3;
  float* pj = part + kPartFloats<D>;       // [rows][ld] P over query blocks, zero past T
  float* sj = pj + (size_t)a.rows * ld;    // [rows][ld] dS, zero past T
  const int bh = blockIdx.x, j0 = blockIdx.y * a.rows;
  const int nr = min(a.rows, a.T - j0);
  const size_t hb = (size_t)bh * a.T * D;
  for (int e = threadIdx.x; e < nr * D; e += kThreads) {
    kc[e] = a.Kc[hb + (size_t)j0 * D + e];
    vc[e] = a.Vc[hb + (size_t)j0 * D + e];
  }
  __syncthreads();
  // one query block per thread: its Qc and dO rows against all nr key blocks
  for (int i = threadIdx.x; i < ld; i += kThreads) {
    float s[kRows], dp[kRows];
    float2 st = make_float2(0.f, 0.f);
    if (i < a.T) {
      row_dots<D>(kc, nr, a.Qc + hb + (size_t)i * D, s);
      row_dots<D>(vc, nr, a.dO + hb + (size_t)i * D, dp);
      st = a.stat[(size_t)bh * a.T + i];
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      if (r < nr) {
        const float p = i < a.T ? exp2f(s[r] * a.sl2 - st.x) : 0.f;
        pj[(size_t)r * ld + i] = p;
        sj[(size_t)r * ld + i] = i < a.T ? p * (dp[r] - st.y) : 0.f;
      }
    }
  }
  __syncthreads();
  // dKc_r = s sum_i dS_ri Qc_i, dVc_r = sum_i P_ri dO_i
  rows_combine<D>(sj, ld, nr, a.Qc + hb, a.T, kc, part);
  rows_combine<D>(pj, ld, nr, a.dO + hb, a.T, vc, part);
  for (int r = 0; r < nr; ++r) {
    const int2 sp = block_span(j0 + r, a.L_src, a.L_ctx, a.b, a.T_src);
    add_rows<D>(a.dk, (size_t)bh * a.L + sp.x, sp.y, kc + r * D, a.scale / (float)sp.y);
    add_rows<D>(a.dv, (size_t)bh * a.L + sp.x, sp.y, vc + r * D, 1.f / (float)sp.y);
  }
}

// Shared-memory bytes of each kernel for `rows` blocks per CTA.
template <int D>
size_t fwd_smem(int T, int rows) { return (size_t)(kVecFloats<D> + kPartFloats<D> + kRows + (size_t)rows * ((T + 3) & ~3)) * 4; }
template <int D>
size_t kv_smem(int T, int rows) { return (size_t)(kVecFloats<D> + kPartFloats<D> + 2 * (size_t)rows * ((T + 3) & ~3)) * 4; }

constexpr size_t kSmemBudget = 160 * 1024;

template <int D>
static cudaError_t launch_t(const Dims& d, CoarseArgs a, bool backward, cudaStream_t st) {
  static std::atomic<unsigned long long> attr_done{0};   // per template instance
  {
    const cudaError_t e = once_per_device(attr_done, [] {
      cudaError_t r = cudaFuncSetAttribute(coarse_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBudget);
      if (r == cudaSuccess)
        r = cudaFuncSetAttribute(coarse_bwd_q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBudget);
      if (r == cudaSuccess)
        r = cudaFuncSetAttribute(coarse_bwd_kv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBudget);
      return r;
    });
    if (e != cudaSuccess) return e;
  }
  // as many blocks per CTA as the score rows leave room for (at most kRows)
  int rq = kRows;
  while (rq > 1 && fwd_smem<D>(d.T, rq) > kSmemBudget) --rq;
  a.rows = rq;
  const dim3 gq(d.BH, (d.T + rq - 1) / rq);
  if (!backward) {
    coarse_fwd_kernel<D><<<gq, kThreads, fwd_smem<D>(d.T, rq), st>>>(a);
    return cudaGetLastError();
  }
  coarse_bwd_q_kernel<D><<<gq, kThreads, fwd_smem<D>(d.T, rq), st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int rk = kRows;
  while (rk > 1 && kv_smem<D>(d.T, rk) > kSmemBudget) --rk;
  a.rows = rk;
  coarse_bwd_kv_kernel<D><<<dim3(d.BH, (d.T + rk - 1) / rk), kThreads, kv_smem<D>(d.T, rk), st>>>(a);
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
