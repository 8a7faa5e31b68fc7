// Planning kernels of the ISA forward pass: steps (1)-(3) and the exact-block
// choice of step (5) of "Method steps in detail" on the paper.rainbus.top
// summary card of "LIVEditor-14B: Lightning Unified Video Editing via
// In-Context Sparse Attention".
//
//   pool_kernel        step (1): per-segment blocks, fp32 means of Q, K, V
//                      (optionally after the decoupled RoPE of Q and K)
//   ctx_select_kernel  step (2): context importance (source query rows summed
//                      over the source x context region of S), TopK, kept
//                      list, bf16 pooled K/V of the kept blocks
//   rowstats_kernel    step (3): E_i = sum_j softmax(S_i)_j^2 over all T
//                      columns, S = Qc Kc^T * scale in fp32, never stored
//   split_kernel       step (3): rank blocks by E (descending, lower block
//                      sharper on ties) into sharp and flat lists
//   exact_kernel       step (5): the n_exact kept blocks with the largest S
//                      for every flat block, as a list and as a bitmap
#include "isa_common.cuh"

namespace isa {

// ---------------------------------------------------------------------------
// K1: pooling.  grid (T, BH, 3), 256 threads.  Each thread reads 16-byte
// vectors (8 bf16) of D/8-wide row chunks; rows of the block are split over
// 256/(D/8) row groups, reduced through shared memory.  HBM bound.
// ROPE: the Q and K rows are first rotated (decoupled RoPE, rot_pair with the
// (cos, sin) of the token's segment position), written once to q_rot/k_rot
// for the attention, and pooled from those rounded values, so Q and K are
// read once for both steps.  Each vector is read and written by one thread,
// so q_rot/k_rot may be q/k; plain loads then (not the read-only path).
// ---------------------------------------------------------------------------
template <int D, bool ROPE>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                                   const __nv_bfloat16* v, Dims dm, float* Qc, float* Kc,
                                                   float* Vc, RopeArgs rope) {
  constexpr int CH = D / 8;          // 16-byte chunks per row
  constexpr int RG = 256 / CH;       // row groups
  __shared__ float part[RG][D];
  const int blk = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const __nv_bfloat16* X = which == 0 ? q : (which == 1 ? k : v);
  float* out = which == 0 ? Qc : (which == 1 ? Kc : Vc);
  const int2 sp = block_span(blk, dm.L_src, dm.L_ctx, dm.b, dm.T_src);
  const int ch = threadIdx.x % CH, rg = threadIdx.x / CH;
  const size_t first = ((size_t)bh * dm.L + sp.x) * CH + ch;   // this thread's vector of the block's row 0
  const uint4* base = reinterpret_cast<const uint4*>(X) + first;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  constexpr int MAXR = 64 / RG > 0 ? 64 / RG : 1;   // rows per thread for b <= 64
  uint4 buf[MAXR];
  const bool rot = ROPE && which < 2;
#pragma unroll
  for (int i = 0; i < MAXR; ++i) {
    const int r = rg + i * RG;
    if constexpr (ROPE) {
      buf[i] = r < sp.y ? base[(size_t)r * CH] : make_uint4(0, 0, 0, 0);
    } else {
      buf[i] = r < sp.y ? __ldg(base + (size_t)r * CH) : make_uint4(0, 0, 0, 0);
    }
  }
  if (rot) {
    // segment position of the block's first token (blocks never straddle segments)
    const int pos0 = blk < dm.T_src ? sp.x : sp.x - dm.L_src;
    uint4* dst = reinterpret_cast<uint4*>(which == 0 ? rope.q_rot : rope.k_rot) + first;
#pragma unroll
    for (int i = 0; i < MAXR; ++i) {
      const int r = rg + i * RG;
      if (r < sp.y) {
        const float4* tp = reinterpret_cast<const float4*>(rope.tab + (size_t)(pos0 + r) * (D / 2) + 4 * ch);
        const float4 t01 = __ldg(tp), t23 = __ldg(tp + 1);
        buf[i] = make_uint4(rot_pair(buf[i].x, make_float2(t01.x, t01.y)),
                            rot_pair(buf[i].y, make_float2(t01.z, t01.w)),
                            rot_pair(buf[i].z, make_float2(t23.x, t23.y)),
                            rot_pair(buf[i].w, make_float2(t23.z, t23.w)));
        dst[(size_t)r * CH] = buf[i];
      }
    }
  }
#pragma unroll
  for (int i = 0; i < MAXR; ++i) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&buf[i]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rg][ch * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) s += part[g][threadIdx.x];
    out[((size_t)bh * dm.T + blk) * D + threadIdx.x] = s / (float)sp.y;
  }
}

// ---------------------------------------------------------------------------
// K2a: context selection.  grid BH, 256 threads.
// imp[c] = sum_{i < T_src} S[i, T_src + c] = scale * (sum_i Qc_i) . Kc_{T_src+c}
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) ctx_select_kernel(Dims dm, PlanPtrs pp) {
  extern __shared__ float sm[];
  float* qsum = sm;               // [D]
  float* imp = sm + D;            // [T_ctx]
  int* sel = reinterpret_cast<int*>(imp + dm.T_ctx);   // [K_sel]
  __shared__ float part[256];
  __shared__ uint32_t hist[256];   // the selection's radix histogram
  const int bh = blockIdx.x, tid = threadIdx.x;
  const float* Qc = pp.Qc + (size_t)bh * dm.T * D;
  const float* Kc = pp.Kc + (size_t)bh * dm.T * D;
  {
    constexpr int SPLIT = 256 / D;
    const int d = tid % D, part_i = tid / D;
    float s = 0.f;
#pragma unroll 16
    for (int i = part_i; i < dm.T_src; i += SPLIT) s += Qc[(size_t)i * D + d];   // loads in flight, adds in order
    part[tid] = s;
    __syncthreads();
    if (tid < D) {
      float t = 0.f;
      for (int p = 0; p < SPLIT; ++p) t += part[p * D + tid];
      qsum[tid] = t;
    }
    __syncthreads();
  }
  const int warp = tid >> 5, lane = tid & 31;
  // four context blocks per warp at a time, so that their Kc rows are
  // fetched together (each dot product keeps its own order of additions)
  constexpr int CR = 4, PER = D / 32;
  for (int c0 = warp * CR; c0 < dm.T_ctx; c0 += 8 * CR) {
    float kv[CR][PER];
#pragma unroll
    for (int u = 0; u < CR; ++u) {
      const float* kr = Kc + (size_t)(dm.T_src + min(c0 + u, dm.T_ctx - 1)) * D;
#pragma unroll
      for (int e = 0; e < PER; ++e) kv[u][e] = kr[lane + 32 * e];
    }
    float s[CR];
#pragma unroll
    for (int u = 0; u < CR; ++u) {
      s[u] = 0.f;
#pragma unroll
      for (int e = 0; e < PER; ++e) s[u] += qsum[lane + 32 * e] * kv[u][e];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < CR; ++u) s[u] += __shfl_xor_sync(0xFFFFFFFFu, s[u], o);
    if (lane < CR && c0 + lane < dm.T_ctx) {
      float v = s[0];
#pragma unroll
      for (int u = 1; u < CR; ++u) v = lane == u ? s[u] : v;
      imp[c0 + lane] = v * dm.scale;
      pp.imp[(size_t)bh * dm.T_ctx + c0 + lane] = v * dm.scale;
    }
  }
  __syncthreads();
  if (warp == 0) warp_topk(imp, dm.T_ctx, dm.K_sel, sel, nullptr, hist);
  __syncthreads();
  int* kept = pp.kept + (size_t)bh * dm.T_kv;
  for (int i = tid; i < dm.K_sel; i += 256) pp.ctx_sel[(size_t)bh * dm.K_sel + i] = sel[i];
  for (int i = tid; i < dm.T_kv; i += 256) kept[i] = i < dm.T_src ? i : dm.T_src + sel[i - dm.T_src];
}

// ---------------------------------------------------------------------------
// K2a': bf16 pooled K and V of the kept blocks (the keys and values of the
// pooled terms), zero rows up to T_kv_pad.  grid (ceil(T_kv_pad/8), BH), 256
// threads; warp w converts kept row 8*blockIdx.x + w, each lane D/32
// consecutive columns.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) pooled_kv_kernel(Dims dm, PlanPtrs pp) {
  const int bh = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;
  if (r >= dm.T_kv_pad) return;
  constexpr int PER = D / 32;
  float kv[PER], vv[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) kv[u] = vv[u] = 0.f;
  if (r < dm.T_kv) {
    const int j = pp.kept[(size_t)bh * dm.T_kv + r];
    const float* kr = pp.Kc + ((size_t)bh * dm.T + j) * D + PER * lane;
    const float* vr = pp.Vc + ((size_t)bh * dm.T + j) * D + PER * lane;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      kv[u] = kr[u];
      vv[u] = vr[u];
    }
  }
  __nv_bfloat16* Kp = pp.Kp + ((size_t)bh * dm.T_kv_pad + r) * D + PER * lane;
  __nv_bfloat16* Vp = pp.Vp + ((size_t)bh * dm.T_kv_pad + r) * D + PER * lane;
#pragma unroll
  for (int u = 0; u < PER; u += 2) {
    *reinterpret_cast<__nv_bfloat162*>(Kp + u) = __floats2bfloat162_rn(kv[u], kv[u + 1]);
    *reinterpret_cast<__nv_bfloat162*>(Vp + u) = __floats2bfloat162_rn(vv[u], vv[u + 1]);
  }
}

// ---------------------------------------------------------------------------
// K2b: row statistics of S.  grid (ceil(T/64), BH), 256 threads, dynamic
// shared memory 2 * 64 * (D+4) floats.  A 64-row tile of Qc stays in shared
// memory; 64-row tiles of Kc stream through (rows padded by 4 floats so that
// the 8 threads of a quarter warp reading 8 different rows hit 8 different
// 16-byte bank groups).  Thread (ty, tx) owns query rows 4ty..4ty+3 and key
// columns tx, tx+16, tx+32, tx+48; the 16 threads sharing a row group are
// one half warp and reduce row statistics with shuffles.  Online update of
// m = max_j s_ij, z = sum_j e^(s_ij - m), y = sum_j e^(2(s_ij - m)), and
// E_i = y / z^2 at the end.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) rowstats_kernel(Dims dm, PlanPtrs pp) {
  constexpr int LD = D + 4;
  extern __shared__ __align__(16) float rs_sm[];
  float* Qs = rs_sm;              // [64][LD]
  float* Ks = rs_sm + 64 * LD;    // [64][LD]
  const int bh = blockIdx.y, i0 = blockIdx.x * 64, tid = threadIdx.x;
  const float* Qc = pp.Qc + (size_t)bh * dm.T * D;
  const float* Kc = pp.Kc + (size_t)bh * dm.T * D;
  constexpr int V4 = D / 4;       // float4 per row
  for (int e = tid; e < 64 * V4; e += 256) {
    const int r = e / V4, c4 = e % V4;
    const float4 val = (i0 + r < dm.T) ? *reinterpret_cast<const float4*>(Qc + (size_t)(i0 + r) * D + 4 * c4)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(Qs + r * LD + 4 * c4) = val;
  }
  const int ty = tid >> 4, tx = tid & 15;
  float m[4], z[4], y[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    m[a] = -INFINITY;
    z[a] = 0.f;
    y[a] = 0.f;
  }
  for (int j0 = 0; j0 < dm.T; j0 += 64) {
    __syncthreads();
    for (int e = tid; e < 64 * V4; e += 256) {
      const int r = e / V4, c4 = e % V4;
      const float4 val = (j0 + r < dm.T) ? *reinterpret_cast<const float4*>(Kc + (size_t)(j0 + r) * D + 4 * c4)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(Ks + r * LD + 4 * c4) = val;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 4
    for (int d = 0; d < D; d += 4) {
      float4 qa[4], kb[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) qa[a] = *reinterpret_cast<const float4*>(Qs + (ty * 4 + a) * LD + d);
#pragma unroll
      for (int c = 0; c < 4; ++c) kb[c] = *reinterpret_cast<const float4*>(Ks + (tx + 16 * c) * LD + d);
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
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float cm = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[a][c] = (j0 + tx + 16 * c < dm.T) ? acc[a][c] * dm.scale : -INFINITY;
        cm = fmaxf(cm, acc[a][c]);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, o));
      const float mn = fmaxf(m[a], cm);
      float ez = 0.f, ey = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float e = expf(acc[a][c] - mn);
        ez += e;
        ey += e * e;
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        ez += __shfl_xor_sync(0xFFFFFFFFu, ez, o);
        ey += __shfl_xor_sync(0xFFFFFFFFu, ey, o);
      }
      const float f = expf(m[a] - mn);     // m = -inf on the first tile -> 0
      z[a] = z[a] * f + ez;
      y[a] = y[a] * f * f + ey;
      m[a] = mn;
    }
  }
  if (tx == 0) {
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int i = i0 + ty * 4 + a;
      if (i < dm.T) pp.energy[(size_t)bh * dm.T + i] = y[a] / (z[a] * z[a]);
    }
  }
}

// ---------------------------------------------------------------------------
// K2c: sharp/flat split.  grid BH, 256 threads; warp 0 selects the n_sharp
// blocks of largest E (ties to the lower block), the rest are flat.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) split_kernel(Dims dm, PlanPtrs pp) {
  extern __shared__ float sm[];
  float* E = sm;                                  // [T]
  int* sharp = reinterpret_cast<int*>(E + dm.T);  // [n_sharp]
  uint32_t* bits = reinterpret_cast<uint32_t*>(sharp + dm.n_sharp);   // [ceil(T/32)]
  __shared__ uint32_t hist[256];   // the selection's radix histogram
  const int bh = blockIdx.x, tid = threadIdx.x;
  for (int i = tid; i < dm.T; i += 256) E[i] = pp.energy[(size_t)bh * dm.T + i];
  __syncthreads();
  if (tid < 32) warp_topk(E, dm.T, dm.n_sharp, sharp, bits, hist);
  __syncthreads();
  for (int i = tid; i < dm.n_sharp; i += 256) pp.sharp[(size_t)bh * dm.n_sharp + i] = sharp[i];
  if (tid < 32) {
    // flat = complement of the sharp bitmap, ascending
    const int lane = tid;
    int base = 0;
    for (int i0 = 0; i0 < dm.T; i0 += 32) {
      const int i = i0 + lane;
      const bool fl = i < dm.T && !((bits[i0 >> 5] >> lane) & 1u);
      const uint32_t fm = __ballot_sync(0xFFFFFFFFu, fl);
      if (fl) pp.flat[(size_t)bh * dm.n_flat + base + __popc(fm & ((1u << lane) - 1u))] = i;
      base += __popc(fm);
    }
  }
}

// ---------------------------------------------------------------------------
// K2d: exact-block lists of the flat blocks.  grid (ceil(n_flat/8), BH),
// 256 threads; warp w owns flat block 8*blockIdx.x + w.  The kept rows of Kc
// stream through shared memory 32 at a time (row stride D+4 floats, so the
// 16-byte reads of eight lanes on eight different rows hit different banks);
// lane l of warp w forms the whole dot product of flat row w with kept row
// l of the chunk.  The scores of all kept blocks for the 8 rows are kept in
// shared memory, then each warp selects its row's exact blocks.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) exact_kernel(Dims dm, PlanPtrs pp) {
  extern __shared__ float sm[];
  float* qrows = sm;                 // [8][D]
  float* sc = sm + 8 * D;            // [8][T_kv]
  __shared__ uint32_t hist[8][256];   // each warp's radix histogram
  const int bh = blockIdx.y, f0 = blockIdx.x * 8, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* Qc = pp.Qc + (size_t)bh * dm.T * D;
  const float* Kc = pp.Kc + (size_t)bh * dm.T * D;
  const int* kept = pp.kept + (size_t)bh * dm.T_kv;
  for (int e = tid; e < 8 * D; e += 256) {
    const int r = e / D, d = e % D, f = f0 + r;
    qrows[e] = f < dm.n_flat ? Qc[(size_t)pp.flat[(size_t)bh * dm.n_flat + f] * D + d] : 0.f;
  }
  __syncthreads();
  constexpr int KS = D + 4;         // padded row stride of the Kc chunk
  float* kch = sc + 8 * dm.T_kv;    // [32][KS]
  const float4* q4 = reinterpret_cast<const float4*>(qrows + warp * D);
  // Each thread moves NPT float4 of every 32-row chunk: column col4 of rows
  // r0 + i*RS.  The chunk after the current one is fetched into registers
  // while the current one is used, and the kept indices one chunk earlier
  // still, so the two dependent L2 reads overlap the dot products.
  constexpr int C4 = D / 4, NPT = 32 * C4 / 256, RS = 256 / C4;
  const int col4 = tid % C4, r0 = tid / C4;
  int nidx[NPT];
  float4 w[NPT];
  auto load_idx = [&](int k) {
#pragma unroll
    for (int i = 0; i < NPT; ++i) nidx[i] = k + r0 + i * RS < dm.T_kv ? kept[k + r0 + i * RS] : -1;
  };
  auto load_rows = [&]() {
#pragma unroll
    for (int i = 0; i < NPT; ++i)
      w[i] = nidx[i] >= 0 ? reinterpret_cast<const float4*>(Kc + (size_t)nidx[i] * D)[col4] : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  load_idx(0);
  load_rows();
  load_idx(32);
  for (int k0 = 0; k0 < dm.T_kv; k0 += 32) {
    __syncthreads();   // the previous chunk is consumed
#pragma unroll
    for (int i = 0; i < NPT; ++i) *reinterpret_cast<float4*>(kch + (r0 + i * RS) * KS + 4 * col4) = w[i];
    __syncthreads();
    if (k0 + 32 < dm.T_kv) {
      load_rows();
      load_idx(k0 + 64);
    }
    const float4* k4 = reinterpret_cast<const float4*>(kch + lane * KS);
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
    for (int c4 = 0; c4 < D / 4; c4 += 2) {
      const float4 a = q4[c4], b = k4[c4], a1 = q4[c4 + 1], b1 = k4[c4 + 1];
      s0 = fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, s0))));
      s1 = fmaf(a1.x, b1.x, fmaf(a1.y, b1.y, fmaf(a1.z, b1.z, fmaf(a1.w, b1.w, s1))));
    }
    if (k0 + lane < dm.T_kv) sc[warp * dm.T_kv + k0 + lane] = (s0 + s1) * dm.scale;
  }
  __syncthreads();
  const int f = f0 + warp;
  if (f < dm.n_flat) {
    uint32_t* bits = pp.bits + ((size_t)bh * dm.n_flat + f) * dm.words;
    int* ex = pp.exact + ((size_t)bh * dm.n_flat + f) * dm.n_exact;
    warp_topk(sc + warp * dm.T_kv, dm.T_kv, dm.n_exact, ex, bits, hist[warp]);
  }
}

// ---------------------------------------------------------------------------
// host-side launchers (called from isa_api.cu)
// ---------------------------------------------------------------------------
static size_t rowstats_smem(int D) { return sizeof(float) * 2 * 64 * (D + 4); }
static size_t exact_kernel_smem(const Dims& dm) {
  return sizeof(float) * (8 * ((size_t)dm.D + dm.T_kv) + 32 * ((size_t)dm.D + 4));
}

template <int D>
static cudaError_t launch_plan_d(const Dims& dm, const void* q, const void* k, const void* v, const PlanPtrs& pp,
                                 cudaStream_t st, const RopeArgs* rope) {
  const dim3 pgrid(dm.T, dm.BH, 3);
  const auto* qb = reinterpret_cast<const __nv_bfloat16*>(q);
  const auto* kb = reinterpret_cast<const __nv_bfloat16*>(k);
  const auto* vb = reinterpret_cast<const __nv_bfloat16*>(v);
  if (rope)
    pool_kernel<D, true><<<pgrid, 256, 0, st>>>(qb, kb, vb, dm, pp.Qc, pp.Kc, pp.Vc, *rope);
  else
    pool_kernel<D, false><<<pgrid, 256, 0, st>>>(qb, kb, vb, dm, pp.Qc, pp.Kc, pp.Vc, RopeArgs{});
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t sm_ctx = sizeof(float) * (D + dm.T_ctx) + sizeof(int) * dm.K_sel;
  ctx_select_kernel<D><<<dm.BH, 256, sm_ctx, st>>>(dm, pp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  pooled_kv_kernel<D><<<dim3((dm.T_kv_pad + 7) / 8, dm.BH), 256, 0, st>>>(dm, pp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  rowstats_kernel<D><<<dim3((dm.T + 63) / 64, dm.BH), 256, rowstats_smem(D), st>>>(dm, pp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t sm_split = sizeof(float) * dm.T + sizeof(int) * dm.n_sharp + sizeof(uint32_t) * ((dm.T + 31) / 32);
  split_kernel<<<dm.BH, 256, sm_split, st>>>(dm, pp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (dm.n_flat > 0) {
    exact_kernel<D><<<dim3((dm.n_flat + 7) / 8, dm.BH), 256, exact_kernel_smem(dm), st>>>(dm, pp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Several planning kernels need more than the default 48 KB of dynamic
// shared memory; the limit is raised on each device before its first plan.
static cudaError_t prepare_plan_kernels() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(rowstats_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)rowstats_smem(64))) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(rowstats_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)rowstats_smem(128))) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(exact_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(sizeof(float) * (8 * (64 + kMaxTkv) + 32 * (64 + 4))))) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(exact_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(sizeof(float) * (8 * (128 + kMaxTkv) + 32 * (128 + 4))))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 3 * kMaxT * 4)) !=
      cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(ctx_select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                3 * kMaxT * 4)) != cudaSuccess) return e;
  return cudaFuncSetAttribute(ctx_select_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, 3 * kMaxT * 4);
}

cudaError_t launch_plan(const Dims& dm, const void* q, const void* k, const void* v, const PlanPtrs& pp,
                        cudaStream_t st, const RopeArgs* rope) {
  static std::atomic<unsigned long long> attr_done{0};
  const cudaError_t e = once_per_device(attr_done, prepare_plan_kernels);
  if (e != cudaSuccess) return e;
  return dm.D == 64 ? launch_plan_d<64>(dm, q, k, v, pp, st, rope) : launch_plan_d<128>(dm, q, k, v, pp, st, rope);
}

}  // namespace isa
