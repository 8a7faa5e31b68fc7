// Decoupled rotary position embedding of Q and K (techwalker.com article,
// "Decoupled RoPE": the reference video's position indices restart at 0
// instead of continuing after the source video; summary card, innovation
// (d): source and context each encode positions from 0).
//
// Reading of what the pages leave open: one-dimensional RoPE over the token
// index, theta_i = base^(-2i/D), pair i = components (2i, 2i+1) rotated
// counter-clockwise by position * theta_i.  Token l has position l in the
// source segment and l - L_src in the context segment.
//
// Two launches: a table of (cos, sin) per (segment position, pair) computed
// in double precision (max(L_src, L_ctx) * D/2 entries, a few MB, read back
// from L2), then one streaming pass over Q and K (HBM-bound: every element
// read once and written once).  isa_plan_rope uses the same table and the
// same rotation (rot_pair) inside the pooling pass instead of the second
// launch, so Q and K are read once for both.
#include <algorithm>

#include "isa_common.cuh"

namespace isa {

// tab[pos * (D/2) + i] = (cos, sin)(pos * base^(-2i/D)), angles in double.
__global__ void __launch_bounds__(256) rope_table_kernel(float2* __restrict__ tab, int n_pos, int D, double base) {
  const int half = D / 2;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n_pos * half) return;
  const int pos = e / half, i = e % half;
  const double theta = pow(base, -2.0 * (double)i / (double)D);
  double s, c;
  sincos((double)pos * theta, &s, &c);
  tab[e] = make_float2((float)c, (float)s);
}

// One thread per 8 consecutive components (4 pairs) of one token row, for
// Q and K together; grid-stride loop over the B*H*L*D/8 vectors.  The
// outputs may be the inputs (each vector is read and written by one thread).
__global__ void __launch_bounds__(256) rope_apply_kernel(const uint4* q, const uint4* k,
                                                         uint4* qo, uint4* ko, const float2* __restrict__ tab,
                                                         size_t n_vec, int L, int L_src, int D) {
  const int vpr = D / 8;   // vectors per row
  for (size_t v = (size_t)blockIdx.x * blockDim.x + threadIdx.x; v < n_vec; v += (size_t)gridDim.x * blockDim.x) {
    const size_t row = v / vpr;
    const int c8 = (int)(v - row * vpr);
    const int l = (int)(row % (size_t)L);
    const int pos = l < L_src ? l : l - L_src;
    const float4* tp = reinterpret_cast<const float4*>(tab + (size_t)pos * (D / 2) + 4 * c8);
    const float4 t01 = __ldg(tp), t23 = __ldg(tp + 1);
    const float2 cs[4] = {make_float2(t01.x, t01.y), make_float2(t01.z, t01.w), make_float2(t23.x, t23.y),
                          make_float2(t23.z, t23.w)};
    const uint4 xq = q[v], xk = k[v];
    qo[v] = make_uint4(rot_pair(xq.x, cs[0]), rot_pair(xq.y, cs[1]), rot_pair(xq.z, cs[2]), rot_pair(xq.w, cs[3]));
    ko[v] = make_uint4(rot_pair(xk.x, cs[0]), rot_pair(xk.y, cs[1]), rot_pair(xk.z, cs[2]), rot_pair(xk.w, cs[3]));
  }
}

size_t rope_table_bytes(const Dims& d) { return (size_t)std::max(d.L_src, d.L_ctx) * (d.D / 2) * sizeof(float2); }

cudaError_t launch_rope_table(const Dims& d, double base, void* tab, cudaStream_t st) {
  const int n_pos = std::max(d.L_src, d.L_ctx);
  const int n_tab = n_pos * (d.D / 2);
  rope_table_kernel<<<(n_tab + 255) / 256, 256, 0, st>>>(static_cast<float2*>(tab), n_pos, d.D, base);
  return cudaGetLastError();
}

cudaError_t launch_rope(const Dims& d, double base, const void* q, const void* k, void* qo, void* ko, void* tab,
                        int sm_count, cudaStream_t st) {
  cudaError_t e = launch_rope_table(d, base, tab, st);
  if (e != cudaSuccess) return e;
  const size_t n_vec = (size_t)d.BH * d.L * (d.D / 8);
  const size_t want = (n_vec + 255) / 256;
  const int grid = (int)std::min<size_t>(want, (size_t)sm_count * 16);
  if (grid == 0) return cudaSuccess;
  rope_apply_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4*>(q), static_cast<const uint4*>(k),
                                           static_cast<uint4*>(qo), static_cast<uint4*>(ko),
                                           static_cast<const float2*>(tab), n_vec, d.L, d.L_src, d.D);
  return cudaGetLastError();
}

}  // namespace isa
