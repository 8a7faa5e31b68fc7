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
// The work is dense attention over the T pooled blocks of a head (T x T x D),
// kept in fp32 on the CUDA cores: the pooled means are fp32, and a bf16
// tensor-core product would round the logits far beyond the residual's
// tolerance.  Each CTA (256 threads) takes 64 query (or key) blocks and walks
// the other side in tiles of 64 rows staged in shared memory; a thread owns a
// 4 x 4 micro-tile of each 64 x 64 score tile (rows 4 ty .. 4 ty + 3, columns
// tx, tx + 16, tx + 32, tx + 48) and 4 rows x D/16 columns of each 64 x D
// product; softmax rows run online (running maximum and sum), as in flash
// attention.  The backward kernels copy the next tile pair in with cp.async
// while they use the current one (one CTA per SM either way); the forward
// keeps one pair, so that two CTAs fit on an SM:
//   coarse_fwd_kernel    O_coarse of 64 query blocks -> out rows += gamma O_i
//   coarse_bwd_q_kernel  per query block i: the forward again (lse2_i, O_i),
//                        dO_i = gamma * sum of the block's dout rows, Delta_i =
//                        dO_i . O_i, dgamma += (dout sum) . O_i; then dS_ij =
//                        P_ij (dO_i . Vc_j - Delta_i), dQc_i = s sum_j dS_ij Kc_j
//                        -> dq rows += dQc_i / n_i; keeps (lse2_i, Delta_i) and
//                        dO_i for the key pass
//   coarse_bwd_kv_kernel per key block j: dKc_j = s sum_i dS_ij Qc_i,
//                        dVc_j = sum_i P_ij dO_i -> dk, dv rows += (.) / n_j
// Gradients reach the tokens through the pooled means (Kc_j is the mean of
// block j's n_j keys), as in the sparse path's backward.
#include "isa_common.cuh"

namespace isa {
namespace coarse {

constexpr int kThreads = 256;
constexpr int kBM = 64;   // blocks per CTA and per tile
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Tile {
  static constexpr int LD = D + 4;              // row stride (floats) of a 64 x D operand tile
  static constexpr int LP = kBM + 4;            // row stride of a 64 x 64 weight tile
  static constexpr int OP = kBM * LD;           // floats of an operand tile
  static constexpr int WP = kBM * LP;           // floats of a weight tile
  static constexpr int NC = D / 16;             // product columns per thread
};

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

// Xs (64 x LD) = rows [r0, r0 + 64) of X (fp32 [n, D]), zero past n.
template <int D>
__device__ void load_tile(float* Xs, const float* __restrict__ X, int r0, int n) {
  constexpr int V4 = D / 4;
  for (int e = threadIdx.x; e < kBM * V4; e += kThreads) {
    const int r = e / V4, c4 = e % V4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < n) v = *reinterpret_cast<const float4*>(X + (size_t)(r0 + r) * D + 4 * c4);
    *reinterpret_cast<float4*>(Xs + r * Tile<D>::LD + 4 * c4) = v;
  }
}

// The same as an asynchronous copy (cp.async, 16 bytes a piece; rows past n
// are filled with zeros by a source size of 0).  The caller commits the
// group and waits for it.
template <int D>
__device__ __forceinline__ void load_tile_async(float* Xs, const float* __restrict__ X, int r0, int n) {
  constexpr int V4 = D / 4;
  for (int e = threadIdx.x; e < kBM * V4; e += kThreads) {
    const int r = e / V4, c4 = e % V4;
    const bool ok = r0 + r < n;
    const float* src = X + (size_t)(ok ? r0 + r : 0) * D + 4 * c4;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(Xs + r * Tile<D>::LD + 4 * c4)),
                 "l"(src), "r"(ok ? 16 : 0)
                 : "memory");
  }
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// waits until at most N of this thread's committed groups are pending
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// acc[a][c] = A[4 ty + a] . B[tx + 16 c] over D (A, B: 64 x LD tiles)
template <int D>
__device__ __forceinline__ void tile_dots(const float* A, const float* B, float (&acc)[4][4]) {
  constexpr int LD = Tile<D>::LD;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 4
  for (int d = 0; d < D; d += 4) {
    float4 qa[4], kb[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) qa[a] = *reinterpret_cast<const float4*>(A + (4 * ty + a) * LD + d);
#pragma unroll
    for (int c = 0; c < 4; ++c) kb[c] = *reinterpret_cast<const float4*>(B + (tx + 16 * c) * LD + d);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[a][c] = fmaf(qa[a].x, kb[c].x, acc[a][c]);
        acc[a][c] = fmaf(qa[a].y, kb[c].y, acc[a][c]);
        acc[a][c] = fmaf(qa[a].z, kb[c].z, acc[a][c]);
        acc[a][c] = fmaf(qa[a].w, kb[c].w, acc[a][c]);
      }
  }
}

// acc[a][n] += sum_k W[4 ty + a][k] X[k][col n]: W a 64 x LP weight tile, X a
// 64 x LD operand tile; this thread's columns are 4 tx + 64 g + (0..3)
template <int D>
__device__ __forceinline__ void tile_mul(const float* W, const float* X, float (&acc)[4][Tile<D>::NC]) {
  constexpr int LD = Tile<D>::LD, LP = Tile<D>::LP, NG = D / 64;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll 2
  for (int k = 0; k < kBM; k += 4) {
    float4 w[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) w[a] = *reinterpret_cast<const float4*>(W + (4 * ty + a) * LP + k);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const float4 x = *reinterpret_cast<const float4*>(X + (k + kk) * LD + 4 * tx + 64 * g);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const float wv = kk == 0 ? w[a].x : kk == 1 ? w[a].y : kk == 2 ? w[a].z : w[a].w;
          acc[a][4 * g + 0] = fmaf(wv, x.x, acc[a][4 * g + 0]);
          acc[a][4 * g + 1] = fmaf(wv, x.y, acc[a][4 * g + 1]);
          acc[a][4 * g + 2] = fmaf(wv, x.z, acc[a][4 * g + 2]);
          acc[a][4 * g + 3] = fmaf(wv, x.w, acc[a][4 * g + 3]);
        }
      }
    }
  }
}

// W[4 ty + a][tx + 16 c] = v[a][c]
template <int D>
__device__ __forceinline__ void store_weights(float* W, const float (&v)[4][4]) {
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) W[(4 * ty + a) * Tile<D>::LP + tx + 16 * c] = v[a][c];
}

// x over the 16 threads of a micro-tile row (lanes 16 (ty & 1) + tx)
__device__ __forceinline__ float row_max16(float x) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xFFFFFFFFu, x, o));
  return x;
}
__device__ __forceinline__ float row_sum16(float x) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
  return x;
}

// The forward of this CTA's 64 query rows (Qs) over all T keys, one (K, V)
// tile pair at a time: running maximum m and sum l (log2 units) per row and
// the unnormalised O.  Uses Ks (then the weight tile) and Vs as scratch.
// The forward kernel takes this form: with one tile pair it holds 99 KB of
// shared memory at D=128 and two CTAs fit on an SM, which beat one CTA with
// the next pair prefetched.
template <int D>
__device__ void flash_rows_sync(const CoarseArgs& a, size_t hb, const float* Qs, float* Ks, float* Vs, float (&m)[4],
                           float (&l)[4], float (&O)[4][Tile<D>::NC]) {
  const int tx = threadIdx.x & 15;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int n = 0; n < Tile<D>::NC; ++n) O[r][n] = 0.f;
  }
  for (int j0 = 0; j0 < a.T; j0 += kBM) {
    __syncthreads();   // the previous tile's readers are done
    load_tile<D>(Ks, a.Kc + hb, j0, a.T);
    load_tile<D>(Vs, a.Vc + hb, j0, a.T);
    __syncthreads();
    float s[4][4];
    tile_dots<D>(Qs, Ks, s);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float cm = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        s[r][c] = (j0 + tx + 16 * c < a.T) ? s[r][c] * a.sl2 : -INFINITY;
        cm = fmaxf(cm, s[r][c]);
      }
      const float mn = fmaxf(m[r], row_max16(cm));   // finite: key j0 + 0 < T
      const float alpha = exp2f(m[r] - mn);           // 0 on the first tile
      float ps = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        s[r][c] = exp2f(s[r][c] - mn);
        ps += s[r][c];
      }
      l[r] = l[r] * alpha + row_sum16(ps);
      m[r] = mn;
#pragma unroll
      for (int n = 0; n < Tile<D>::NC; ++n) O[r][n] *= alpha;
    }
    __syncthreads();   // every thread has read Ks: the weights take its place
    store_weights<D>(Ks, s);
    __syncthreads();
    tile_mul<D>(Ks, Vs, O);
  }
}

// The forward of this CTA's 64 query rows (Qs) over all T keys: running
// maximum m and sum l (log2 units) per row and the unnormalised O.  KV holds
// two (K, V) tile pairs: the next pair is copied in while the current one is
// used, and the current K tile takes the weights once its scores are formed.
template <int D>
__device__ void flash_rows(const CoarseArgs& a, size_t hb, const float* Qs, float* KV, float (&m)[4], float (&l)[4],
                           float (&O)[4][Tile<D>::NC]) {
  using C = Tile<D>;
  const int tx = threadIdx.x & 15;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int n = 0; n < C::NC; ++n) O[r][n] = 0.f;
  }
  __syncthreads();   // the buffers' previous users are done
  load_tile_async<D>(KV, a.Kc + hb, 0, a.T);
  load_tile_async<D>(KV + C::OP, a.Vc + hb, 0, a.T);
  cp_async_commit();
  for (int j0 = 0, u = 0; j0 < a.T; j0 += kBM, u ^= 1) {
    float* Ks = KV + 2 * u * C::OP;
    float* Vs = Ks + C::OP;
    if (j0 + kBM < a.T) {   // the next pair into the other buffers (free since the end of the last tile)
      load_tile_async<D>(KV + 2 * (u ^ 1) * C::OP, a.Kc + hb, j0 + kBM, a.T);
      load_tile_async<D>(KV + (2 * (u ^ 1) + 1) * C::OP, a.Vc + hb, j0 + kBM, a.T);
    }
    cp_async_commit();
    cp_async_wait<1>();   // this tile's pair has landed (this thread's part)
    __syncthreads();      // and every thread's
    float s[4][4];
    tile_dots<D>(Qs, Ks, s);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float cm = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        s[r][c] = (j0 + tx + 16 * c < a.T) ? s[r][c] * a.sl2 : -INFINITY;
        cm = fmaxf(cm, s[r][c]);
      }
      const float mn = fmaxf(m[r], row_max16(cm));   // finite: key j0 + 0 < T
      const float alpha = exp2f(m[r] - mn);           // 0 on the first tile
      float ps = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        s[r][c] = exp2f(s[r][c] - mn);
        ps += s[r][c];
      }
      l[r] = l[r] * alpha + row_sum16(ps);
      m[r] = mn;
#pragma unroll
      for (int n = 0; n < C::NC; ++n) O[r][n] *= alpha;
    }
    __syncthreads();   // every thread has read Ks: the weights take its place
    store_weights<D>(Ks, s);
    __syncthreads();
    tile_mul<D>(Ks, Vs, O);
    __syncthreads();   // the pair's buffers may take the pair after next
  }
  cp_async_wait<0>();
}

// Xs (64 x LD) = the thread's 4 x NC values (rows 4 ty + r, columns 4 tx + 64 g + i)
template <int D>
__device__ __forceinline__ void stage_rows(float* Xs, const float (&v)[4][Tile<D>::NC]) {
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int g = 0; g < D / 64; ++g)
      *reinterpret_cast<float4*>(Xs + (4 * ty + r) * Tile<D>::LD + 4 * tx + 64 * g) =
          make_float4(v[r][4 * g], v[r][4 * g + 1], v[r][4 * g + 2], v[r][4 * g + 3]);
}

// rows [t0, t0 + n) of x (bf16 [.., D]) += scale * v (fp32 [D] in shared memory)
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

template <int D>
__global__ void __launch_bounds__(kThreads) coarse_fwd_kernel(const CoarseArgs a) {
  using C = Tile<D>;
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;
  float* Ks = Qs + C::OP;   // K tile, then the weights; finally O_coarse rows
  float* Vs = Ks + C::OP;
  const int bh = blockIdx.y, i0 = blockIdx.x * kBM;
  const int nr = min(kBM, a.T - i0);
  const size_t hb = (size_t)bh * a.T * D;
  load_tile<D>(Qs, a.Qc + hb, i0, a.T);
  float m[4], l[4], O[4][C::NC];
  flash_rows_sync<D>(a, hb, Qs, Ks, Vs, m, l, O);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float inv = 1.f / l[r];
#pragma unroll
    for (int n = 0; n < C::NC; ++n) O[r][n] *= inv;
  }
  __syncthreads();
  stage_rows<D>(Ks, O);
  __syncthreads();
  for (int r = 0; r < nr; ++r) {
    const int2 sp = block_span(i0 + r, a.L_src, a.L_ctx, a.b, a.T_src);
    add_rows<D>(a.out, (size_t)bh * a.L + sp.x, sp.y, Ks + r * C::LD, a.gamma);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) coarse_bwd_q_kernel(const CoarseArgs a) {
  using C = Tile<D>;
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;
  float* dOs = Qs + C::OP;   // dout block sums, then gamma * them
  float* KV = dOs + C::OP;   // two (K, V) tile pairs
  float* Ws = KV + 4 * C::OP;   // dS tile
  __shared__ float2 st[kBM];   // (lse2, Delta) of the CTA's rows
  const int bh = blockIdx.y, i0 = blockIdx.x * kBM;
  const int nr = min(kBM, a.T - i0);
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  const size_t hb = (size_t)bh * a.T * D;
  load_tile<D>(Qs, a.Qc + hb, i0, a.T);
  // block sums of dout: one (row, 8-column group) at a time, zero past T
  for (int e = threadIdx.x; e < kBM * (D / 8); e += kThreads) {
    const int r = e / (D / 8), c = (e % (D / 8)) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (r < nr) {
      const int2 sp = block_span(i0 + r, a.L_src, a.L_ctx, a.b, a.T_src);
      const __nv_bfloat16* src = a.dout + ((size_t)bh * a.L + sp.x) * D + c;
      for (int t = 0; t < sp.y; ++t) {
        const uint4 w = *reinterpret_cast<const uint4*>(src + (size_t)t * D);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(h[k]);
          acc[2 * k] += f.x;
          acc[2 * k + 1] += f.y;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) dOs[r * C::LD + c + k] = acc[k];
  }
  // the forward again: lse2 and O of the CTA's rows
  float m[4], l[4], O[4][C::NC];
  flash_rows<D>(a, hb, Qs, KV, m, l, O);
  __syncthreads();   // dOs complete
  float lse2[4], delta[4];
  float gsum = 0.f;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float inv = 1.f / l[r];
    lse2[r] = m[r] + __log2f(l[r]);
    float g = 0.f;
#pragma unroll
    for (int gg = 0; gg < D / 64; ++gg)
#pragma unroll
      for (int i = 0; i < 4; ++i) g = fmaf(dOs[(4 * ty + r) * C::LD + 4 * tx + 64 * gg + i], O[r][4 * gg + i] * inv, g);
    g = row_sum16(g);   // (sum of the block's dout rows) . O_coarse
    delta[r] = a.gamma * g;
    if (4 * ty + r < nr) gsum += g;
    if (tx == 0) st[4 * ty + r] = make_float2(lse2[r], delta[r]);
  }
  if (a.dgamma && tx == 0 && gsum != 0.f) atomicAdd(a.dgamma + bh, gsum);
  __syncthreads();
  // dO = gamma * sums, kept for the key pass with (lse2, Delta)
  for (int e = threadIdx.x; e < kBM * D; e += kThreads) {
    const int r = e / D, c = e % D;
    const float x = a.gamma * dOs[r * C::LD + c];
    dOs[r * C::LD + c] = x;
    if (r < nr) a.dO[hb + (size_t)(i0 + r) * D + c] = x;
  }
  for (int r = threadIdx.x; r < nr; r += kThreads) a.stat[(size_t)bh * a.T + i0 + r] = st[r];
  // dQc = s sum_j dS_j Kc_j
  float dQ[4][C::NC];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int n = 0; n < C::NC; ++n) dQ[r][n] = 0.f;
  __syncthreads();   // dOs scaled; the flash pass's buffers are free
  load_tile_async<D>(KV, a.Kc + hb, 0, a.T);
  load_tile_async<D>(KV + C::OP, a.Vc + hb, 0, a.T);
  cp_async_commit();
  for (int j0 = 0, u = 0; j0 < a.T; j0 += kBM, u ^= 1) {
    float* Ks = KV + 2 * u * C::OP;
    float* Vs = Ks + C::OP;
    if (j0 + kBM < a.T) {
      load_tile_async<D>(KV + 2 * (u ^ 1) * C::OP, a.Kc + hb, j0 + kBM, a.T);
      load_tile_async<D>(KV + (2 * (u ^ 1) + 1) * C::OP, a.Vc + hb, j0 + kBM, a.T);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    float s[4][4], dp[4][4];
    tile_dots<D>(Qs, Ks, s);
    tile_dots<D>(dOs, Vs, dp);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float p = (j0 + tx + 16 * c < a.T) ? exp2f(s[r][c] * a.sl2 - lse2[r]) : 0.f;
        s[r][c] = p * (dp[r][c] - delta[r]);
      }
    store_weights<D>(Ws, s);
    __syncthreads();
    tile_mul<D>(Ws, Ks, dQ);
    __syncthreads();   // Ws and this pair's buffers are free again
  }
  cp_async_wait<0>();
  stage_rows<D>(KV, dQ);
  __syncthreads();
  for (int r = 0; r < nr; ++r) {
    const int2 sp = block_span(i0 + r, a.L_src, a.L_ctx, a.b, a.T_src);
    add_rows<D>(a.dq, (size_t)bh * a.L + sp.x, sp.y, KV + r * C::LD, a.scale / (float)sp.y);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) coarse_bwd_kv_kernel(const CoarseArgs a) {
  using C = Tile<D>;
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;            // this CTA's 64 key blocks (stationary); finally dKc rows
  float* Vs = Ks + C::OP;    // their values; finally dVc rows
  float* QD = Vs + C::OP;    // two (Qc, gamma * dout sums) tile pairs of 64 query blocks
  float* Ws = QD + 4 * C::OP;   // P^T, then dS^T [key][query]
  __shared__ float2 st[2][kBM];
  const int bh = blockIdx.y, j0 = blockIdx.x * kBM;
  const int nr = min(kBM, a.T - j0);
  const int tx = threadIdx.x & 15;
  const size_t hb = (size_t)bh * a.T * D;
  load_tile<D>(Ks, a.Kc + hb, j0, a.T);
  load_tile<D>(Vs, a.Vc + hb, j0, a.T);
  float dK[4][C::NC], dV[4][C::NC];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int n = 0; n < C::NC; ++n) dK[r][n] = dV[r][n] = 0.f;
  auto load_pair = [&](int i0, int u) {
    load_tile_async<D>(QD + 2 * u * C::OP, a.Qc + hb, i0, a.T);
    load_tile_async<D>(QD + (2 * u + 1) * C::OP, a.dO + hb, i0, a.T);
    for (int r = threadIdx.x; r < kBM; r += kThreads) {
      const bool ok = i0 + r < a.T;
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(&st[u][r])),
                   "l"(a.stat + (size_t)bh * a.T + (ok ? i0 + r : 0)), "r"(ok ? 8 : 0)
                   : "memory");
    }
  };
  load_pair(0, 0);
  cp_async_commit();
  for (int i0 = 0, u = 0; i0 < a.T; i0 += kBM, u ^= 1) {
    const float* Qs = QD + 2 * u * C::OP;
    const float* dOs = Qs + C::OP;
    if (i0 + kBM < a.T) load_pair(i0 + kBM, u ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    float s[4][4], dp[4][4];
    tile_dots<D>(Ks, Qs, s);    // S^T: key rows, query columns tx + 16 c
    tile_dots<D>(Vs, dOs, dp);  // dP^T
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int qi = tx + 16 * c;
        const float2 q = st[u][qi];
        const float p = i0 + qi < a.T ? exp2f(s[r][c] * a.sl2 - q.x) : 0.f;
        s[r][c] = p;
        dp[r][c] = p * (dp[r][c] - q.y);
      }
    store_weights<D>(Ws, s);
    __syncthreads();
    tile_mul<D>(Ws, dOs, dV);
    __syncthreads();   // P^T read: dS^T takes its place
    store_weights<D>(Ws, dp);
    __syncthreads();
    tile_mul<D>(Ws, Qs, dK);
    __syncthreads();   // this pair's buffers and Ws are free again
  }
  cp_async_wait<0>();
  __syncthreads();
  stage_rows<D>(Ks, dK);
  stage_rows<D>(Vs, dV);
  __syncthreads();
  for (int r = 0; r < nr; ++r) {
    const int2 sp = block_span(j0 + r, a.L_src, a.L_ctx, a.b, a.T_src);
    add_rows<D>(a.dk, (size_t)bh * a.L + sp.x, sp.y, Ks + r * C::LD, a.scale / (float)sp.y);
    add_rows<D>(a.dv, (size_t)bh * a.L + sp.x, sp.y, Vs + r * C::LD, 1.f / (float)sp.y);
  }
}

template <int D>
constexpr size_t fwd_smem() { return (size_t)3 * Tile<D>::OP * 4; }
template <int D>
constexpr size_t bwd_q_smem() { return ((size_t)6 * Tile<D>::OP + Tile<D>::WP) * 4; }
template <int D>
constexpr size_t bwd_kv_smem() { return ((size_t)6 * Tile<D>::OP + Tile<D>::WP) * 4; }

template <int D>
static cudaError_t launch_t(const Dims& d, CoarseArgs a, bool backward, cudaStream_t st) {
  static std::atomic<unsigned long long> attr_done{0};   // per template instance
  {
    const cudaError_t e = once_per_device(attr_done, [] {
      cudaError_t r = cudaFuncSetAttribute(coarse_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fwd_smem<D>());
      if (r == cudaSuccess)
        r = cudaFuncSetAttribute(coarse_bwd_q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bwd_q_smem<D>());
      if (r == cudaSuccess)
        r = cudaFuncSetAttribute(coarse_bwd_kv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bwd_kv_smem<D>());
      return r;
    });
    if (e != cudaSuccess) return e;
  }
  const dim3 grid((d.T + kBM - 1) / kBM, d.BH);
  if (!backward) {
    coarse_fwd_kernel<D><<<grid, kThreads, fwd_smem<D>(), st>>>(a);
    return cudaGetLastError();
  }
  coarse_bwd_q_kernel<D><<<grid, kThreads, bwd_q_smem<D>(), st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  coarse_bwd_kv_kernel<D><<<grid, kThreads, bwd_kv_smem<D>(), st>>>(a);
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
