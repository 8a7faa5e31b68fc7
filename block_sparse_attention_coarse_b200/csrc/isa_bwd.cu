// Backward of the ISA sparse attention for sm_100a: gradients of steps
// (4)-(6) of "Method steps in detail" (paper.rainbus.top summary card of
// "LIVEditor-14B: Lightning Unified Video Editing via In-Context Sparse
// Attention") with respect to Q, K and V, with the plan held fixed.  The
// pages state that the method has a differentiable forward + backward
// implementation and is trained end to end ("Core method", innovation (c))
// without giving formulas; the gradients here are those of the forward as
// computed: the plan's index sets carry no gradient, and the pooled means
// Kc_j, Vc_j of the flat path pass their gradient to every token of block j
// with weight 1/n_j.
//
// With P the softmax weights of a query row over its columns (exact key
// tokens and, for flat rows, pooled keys with log-weight ln n_j), dP = dO V^T
// and Delta = rowsum(dO * O):
//   dS = P * (dP - Delta),  dQ = s dS K,  dK = s dS^T Q,  dV = P^T dO.
//
// Launches, in stream order:
//   bwd_prep_kernel        Delta and lse*log2(e) per query row, block-padded (HBM-bound)
//   bwd_zero_unkept_kernel dK = dV = 0 for context blocks the pre-selection dropped
//   bwd_kv_kernel (pooled) key/value-stationary over the head's pooled rows:
//                          dKc_j, dVc_j (fp32) from every flat block
//   bwd_kv_kernel (kept)   key/value-stationary over the kept blocks: dK, dV
//                          from the sharp blocks and the flat blocks that
//                          attend the block exactly, plus dKc_j/n_j, dVc_j/n_j
//   bwd_q_kernel           query-stationary over the forward's work items: dQ
// P is recomputed from the forward's lse, so no attention matrix is stored.
#include <algorithm>

#include "isa_common.cuh"
#include "isa_items.cuh"

namespace isa {

namespace bwd {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// per-row preparation
// ---------------------------------------------------------------------------

__device__ __forceinline__ float dot_bf16x8(uint4 a, uint4 b) {
  const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&b);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 fx = __bfloat1622float2(x[i]), fy = __bfloat1622float2(y[i]);
    acc = fmaf(fx.x, fy.x, acc);
    acc = fmaf(fx.y, fy.y, acc);
  }
  return acc;
}

// dl[((bh*T + j)*2 + 0)*b + r] = lse * log2 e and dl[((bh*T + j)*2 + 1)*b + r]
// = sum_d dout * o of row r of block j of head bh, and (inf, 0) for r past
// the block's end: every query block's entries are a run of b lse2 values
// followed by a run of b Delta values.  D/8 lanes per entry,
// grid-stride over the BH*T*b entries (the loop bound is warp-uniform).
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint4* __restrict__ o, const uint4* __restrict__ dout,
                                                       const float* __restrict__ lse, float* __restrict__ dl,
                                                       int T, int b, int L, int L_src, int L_ctx, int T_src,
                                                       size_t entries) {
  constexpr int LPR = D / 8;
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const size_t warp = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const size_t nwarps = ((size_t)gridDim.x * blockDim.x) >> 5;
  for (size_t e0 = warp * RPW; e0 < entries; e0 += nwarps * RPW) {
    const size_t e = e0 + lane / LPR;
    bool valid = false;
    size_t row = 0;
    if (e < entries) {
      const size_t bh = e / ((size_t)T * b);
      const int j = (int)((e / b) % T), r = (int)(e % b);
      const int2 sp = block_span(j, L_src, L_ctx, b, T_src);
      valid = r < sp.y;
      row = bh * L + sp.x + r;
    }
    float acc = 0.f;
    if (valid) acc = dot_bf16x8(o[row * LPR + lane % LPR], dout[row * LPR + lane % LPR]);
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
    if (e < entries && lane % LPR == 0) {
      const size_t blk = e / b, r = e % b;   // (bh*T + j), row in the block
      dl[(blk * 2) * b + r] = valid ? lse[row] * kLog2e : INFINITY;
      dl[(blk * 2 + 1) * b + r] = valid ? acc : 0.f;
    }
  }
}

// dK and dV rows of context block blockIdx.y of head blockIdx.x are zero when
// the pre-selection dropped the block (it takes part in neither path).
__global__ void __launch_bounds__(128) bwd_zero_unkept_kernel(const int* __restrict__ ctx_sel, int K_sel, int L,
                                                              int L_src, int L_ctx, int b, int D, uint4* dk, uint4* dv) {
  const int bh = blockIdx.x, c = blockIdx.y;
  const int* sel = ctx_sel + (size_t)bh * K_sel;
  int lo = 0, hi = K_sel;   // ctx_sel is ascending
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (sel[mid] < c) lo = mid + 1;
    else hi = mid;
  }
  if (lo < K_sel && sel[lo] == c) return;
  const int s = c * b;
  const int n = min(b, L_ctx - s);
  const size_t first = ((size_t)bh * L + L_src + s) * (D / 8);
  const size_t cnt = (size_t)n * (D / 8);
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (size_t i = threadIdx.x; i < cnt; i += blockDim.x) {
    dk[first + i] = z;
    dv[first + i] = z;
  }
}


// ---------------------------------------------------------------------------
// key/value-stationary kernel: dK, dV
// ---------------------------------------------------------------------------
// An item is one 128-row key/value tile of one head and stays in shared
// memory while 128-row query steps stream past it:
//   kept launch   : rows = G = 128/R consecutive kept blocks (kept positions
//                   tile*G ..); steps = every sharp block, then the flat
//                   blocks whose exact list holds one of the tile's blocks
//                   (rows of the other blocks masked per query block)
//   pooled launch : rows = 128 consecutive pooled kept blocks (Kp/Vp rows);
//                   steps = every flat block, with the flat block's own exact
//                   blocks masked out; log-weight log2(n_j) per row
// A step is GQ = 128/R query blocks (128 query columns).  Per step u (TMEM
// lane = key/value row):
//   S^T = K Q^T, dP^T = V dO^T         (SS, M=128, N=128, K=D)
//   P^T = 2^(S^T s log2e + w_j - lse2)                      (softmax, phase A)
//   dS^T = P^T (dP^T - Delta)                               (softmax, phase B)
//   dV += P^T dO, dK += dS^T Q         (TS: P^T / dS^T read as bf16 from TMEM)
// The tensor core runs 128 x 128 k-steps at full rate only from N = 128 up
// (N = 64 takes as long as N = 128), so steps are 128 query rows wide, and
// TMEM then holds one S^T and one dP^T buffer beside dV and dK.  The four
// products of consecutive steps are issued as dV_u, S^T_{u+1}, dK_u,
// dP^T_{u+1}: phase A of step u+1 (the exponentials) runs behind dK_u and
// dP^T_{u+1}, phase B behind dV_{u+1} and S^T_{u+2}.  A product that
// overwrites a buffer is issued after the one that reads it; the tensor
// pipe runs one thread's MMAs in order.
// Roles (576 threads, one CTA per SM): warp 0 producer (the whole warp finds
// the steps; lane 0 loads the tile, publishes each step's metadata and
// issues its copies), warp 1 MMA issuer (converged, one elected lane),
// warps 2..17: warp w owns TMEM lanes 32*(w%4).. and query columns
// 32*((w-2)/4).. of each step (four warps per lane quarter, so that each
// scheduler interleaves four of them), and writes the epilogue.
constexpr int kKvSoft = 16;                      // softmax warps
constexpr int kKvThreads = 64 + 32 * kKvSoft;
constexpr int kNSQ = 2;           // query/dO step stages
// TMEM: S^T then P^T, dP^T then dS^T (each softmax warp packs its bf16
// values of query columns 16k..16k+15 into columns 16k..16k+7 of the fp32
// columns it has just read, where the dV / dK products take them as the A
// operand); then dV and dK.
constexpr uint32_t kTST = 0;      // S^T, then P^T
constexpr uint32_t kTDP = 128;    // dP^T, then dS^T
constexpr uint32_t kTDV = 256;    // dV accumulator (D columns); dK at kTDV + D

template <int D, int R>
struct KvCfg {
  static constexpr int G = 128 / R;               // kept blocks per tile
  static constexpr int GQ = 128 / R;              // query blocks per step
  static constexpr int NCH = D / 64;              // 64-column chunks of a row
  static constexpr uint32_t CHUNK = 128 * 128;    // 128 rows x 128 bytes
  static constexpr uint32_t TILE = 128 * D * 2;   // one 128-row tile (K, V, a Q or a dO step)
  static constexpr uint32_t BOX = R * 128;        // one TMA box
  static constexpr uint32_t K_OFF = 0;
  static constexpr uint32_t V_OFF = TILE;
  static constexpr uint32_t Q_OFF = 2 * TILE;
  static constexpr uint32_t DO_OFF = Q_OFF + kNSQ * TILE;
  static constexpr uint32_t DL_OFF = DO_OFF + kNSQ * TILE;   // lse2 and Delta runs of the step's query blocks
  static constexpr uint32_t DL_STAGE = 128 * 8;
  static constexpr uint32_t SMEM_USED = DL_OFF + kNSQ * DL_STAGE + 1024;
  // at least 120 KB so that one CTA (and one 512-column TMEM allocation) fits on an SM
  static constexpr uint32_t SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t ID_T = idesc_bf16_f32(128, 128, 0);
  static constexpr uint32_t ID_A = idesc_bf16_f32(128, D, 1);
};

struct StepMeta {
  int blk[4];             // block ids of the step's query blocks
  int start[4], cnt[4];   // token start and valid rows of the step's query blocks
  uint32_t m[4][4];       // tile rows each query block attends (bit r of m[g][r/32])
  int last;               // last step of the item
};

__device__ __forceinline__ void clear_meta(StepMeta& m) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    m.blk[g] = 0;
    m.start[g] = 0;
    m.cnt[g] = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) m.m[g][w] = 0u;
  }
  m.last = 0;
}

template <int D, int R>
__global__ void __launch_bounds__(kKvThreads, 1)
    bwd_kv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kp,
                  const __grid_constant__ CUtensorMap tm_vp, const __grid_constant__ CUtensorMap tm_do,
                  const BwdArgs b) {
  using C = KvCfg<D, R>;
  constexpr int G = C::G, GQ = C::GQ;
  static_assert(GQ <= 4, "StepMeta holds four query blocks");
  const AttnArgs& a = b.a;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t kv_full, kv_empty, q_full[kNSQ], q_empty[kNSQ];
  __shared__ __align__(8) uint64_t s_full, dp_full, p_ready, ds_ready;
  __shared__ __align__(8) uint64_t acc_ready, acc_free, drain_bar, inject_bar;
  __shared__ StepMeta meta[kNSQ];
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const bool pooled = b.kv_pooled != 0;

  if (tid == 0) {
    mbar_init(&kv_full, 1);
    mbar_init(&kv_empty, 1);
    for (int i = 0; i < kNSQ; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    mbar_init(&s_full, 1);
    mbar_init(&dp_full, 1);
    mbar_init(&p_ready, kKvSoft);    // one arrival per softmax warp
    mbar_init(&ds_ready, kKvSoft);
    mbar_init(&acc_ready, 1);
    mbar_init(&acc_free, kKvSoft);
    mbar_init(&drain_bar, 1);
    mbar_init(&inject_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(pooled ? &tm_kp : &tm_k);
    tma_prefetch_desc(pooled ? &tm_vp : &tm_v);
  }
  if (warp == 1) tmem_alloc(&tmem_base_sh, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const WaitCtl wc{&abort_flag, a.status, a.timeout_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp finds the steps (32 sharp ids or 32 flat blocks' exact
    // bitmaps per round of loads, matches picked by ballot); lane 0 publishes
    // them and issues every copy.
    int kv_cnt = 0, qcnt[kNSQ];
    for (int i = 0; i < kNSQ; ++i) qcnt[i] = 0;
    int u = 0, n = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < b.kv_total; it += gridDim.x, ++n) {
      const int bh = it / b.kv_tiles, tile = it % b.kv_tiles;
      if (lane == 0) {
        if (n >= 1 && !mbar_wait(&kv_empty, (n - 1) & 1, wc)) {
          ok = false;
        } else {
          mbar_arrive_expect_tx(&kv_full, 2 * C::TILE);
          ++kv_cnt;
          for (int g = 0; g < G; ++g) {
            int row;
            if (pooled) {
              row = bh * a.T_kv_pad + tile * 128 + g * R;
            } else {
              const int kk = tile * G + g;
              row = bh * a.L;
              if (kk < a.T_kv) row += block_span(a.kept[(size_t)bh * a.T_kv + kk], a.L_src, a.L_ctx, a.b, a.T_src).x;
            }
            for (int c = 0; c < C::NCH; ++c) {
              tma_load_2d(sgen + C::K_OFF + c * C::CHUNK + g * C::BOX, pooled ? &tm_kp : &tm_k, c * 64, row, &kv_full);
              tma_load_2d(sgen + C::V_OFF + c * C::CHUNK + g * C::BOX, pooled ? &tm_vp : &tm_v, c * 64, row, &kv_full);
            }
          }
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      // Steps are published one behind, so that the last one can be marked
      // (lane 0's copies of pend/grp are the live ones).
      StepMeta pend, grp;
      bool have = false;
      int ng = 0;
      clear_meta(grp);
      auto emit = [&](const StepMeta& m, int last) -> bool {
        const int s = u % kNSQ;
        if (u >= kNSQ && !mbar_wait(&q_empty[s], ((u / kNSQ) - 1) & 1, wc)) return false;
        meta[s] = m;
        meta[s].last = last;   // published by the arrive below (release), read after q_full (acquire)
        mbar_arrive_expect_tx(&q_full[s], 2 * C::TILE + C::DL_STAGE);
        ++qcnt[s];
        for (int g = 0; g < GQ; ++g) {
          const int row = bh * a.L + (m.cnt[g] > 0 ? m.start[g] : 0);
          bulk_load_1d(sgen + C::DL_OFF + s * C::DL_STAGE + g * R * 8,
                       b.dl + ((size_t)bh * (a.T_src + a.T_ctx) + m.blk[g]) * 2 * R, R * 8, &q_full[s]);
          for (int c = 0; c < C::NCH; ++c) {
            tma_load_2d(sgen + C::Q_OFF + s * C::TILE + c * C::CHUNK + g * C::BOX, &tm_q, c * 64, row, &q_full[s]);
            tma_load_2d(sgen + C::DO_OFF + s * C::TILE + c * C::CHUNK + g * C::BOX, &tm_do, c * 64, row,
                        &q_full[s]);
          }
        }
        ++u;
        return true;
      };
      auto push = [&](const StepMeta& m) -> bool {
        const bool r = have ? emit(pend, 0) : true;
        pend = m;
        have = true;
        return r;
      };
      // query block blk (row mask mw) joins the step being assembled; lane 0 only
      auto add = [&](int blk, const uint32_t (&mw)[4]) -> bool {
        const int2 sp = block_span(blk, a.L_src, a.L_ctx, a.b, a.T_src);
        grp.blk[ng] = blk;
        grp.start[ng] = sp.x;
        grp.cnt[ng] = sp.y;
        for (int w = 0; w < 4; ++w) grp.m[ng][w] = mw[w];
        if (++ng < GQ) return true;
        const bool r = push(grp);
        clear_meta(grp);
        ng = 0;
        return r;
      };
      if (!pooled) {
        // sharp blocks attend every kept block: all rows of the tile
        const uint32_t all[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu};
        for (int base = 0; ok && base < a.n_sharp; base += 32) {
          const int idx = base + lane;
          const int blk = idx < a.n_sharp ? a.sharp[(size_t)bh * a.n_sharp + idx] : 0;
          const int cnt = min(32, a.n_sharp - base);
          for (int j = 0; j < cnt; ++j) {
            const int bj = __shfl_sync(0xFFFFFFFFu, blk, j);
            if (lane == 0) ok = add(bj, all);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
          }
        }
        if (lane == 0 && ok && ng > 0) {   // the sharp blocks' last partial step
          ok = push(grp);
          clear_meta(grp);
          ng = 0;
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      }
      for (int base = 0; ok && base < a.n_flat; base += 32) {
        const int f = base + lane;
        uint32_t mw[4] = {0u, 0u, 0u, 0u};
        int blk = 0;
        if (f < a.n_flat) {
          const uint32_t* fb = a.bits + ((size_t)bh * a.n_flat + f) * a.words;
          if (pooled) {
            // pooled rows tile*128 + r, minus the flat block's exact blocks
            for (int w = 0; w < 4; ++w) {
              const int wi = tile * 4 + w;
              const int rem = a.T_kv - (tile * 128 + 32 * w);
              const uint32_t range = rem >= 32 ? 0xFFFFFFFFu : (rem <= 0 ? 0u : ((1u << rem) - 1u));
              mw[w] = range & ~(wi < a.words ? fb[wi] : 0u);
            }
          } else {
            // exact blocks among kept positions tile*G .. tile*G+G-1 (one word)
            const int k0 = tile * G;
            const uint32_t gm = (fb[k0 >> 5] >> (k0 & 31)) & ((1u << G) - 1u);
            for (int w = 0; w < 4; ++w) mw[w] = ((gm >> ((32 * w) / R)) & 1u) ? 0xFFFFFFFFu : 0u;
          }
          if (mw[0] | mw[1] | mw[2] | mw[3]) blk = a.flat[(size_t)bh * a.n_flat + f];
        }
        uint32_t bal = __ballot_sync(0xFFFFFFFFu, (mw[0] | mw[1] | mw[2] | mw[3]) != 0u);
        while (bal) {
          const int src = __ffs(bal) - 1;
          bal &= bal - 1;
          uint32_t m4[4];
          for (int w = 0; w < 4; ++w) m4[w] = __shfl_sync(0xFFFFFFFFu, mw[w], src);
          const int bj = __shfl_sync(0xFFFFFFFFu, blk, src);
          if (lane == 0) ok = add(bj, m4);
          ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
          if (!ok) break;
        }
      }
      if (lane == 0 && ok) {
        if (ng > 0) ok = push(grp);
        if (ok && !have) {
          clear_meta(pend);   // no query attends the tile: one empty step writes zeros
          have = true;
        }
        if (ok) ok = emit(pend, 1);
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    }
    // let every copy in flight land before the CTA can exit
    if (lane == 0) {
      if (kv_cnt) mbar_wait_drain(&kv_full, (kv_cnt - 1) & 1, a.timeout_ns);
      for (int i = 0; i < kNSQ; ++i)
        if (qcnt[i]) mbar_wait_drain(&q_full[i], (qcnt[i] - 1) & 1, a.timeout_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per step u: dV_u (needs P^T_u), S^T_{u+1} (overwrites P^T_u), dK_u
    // (needs dS^T_u), dP^T_{u+1} (overwrites dS^T_u).  One commit per product
    // group that someone waits for.
    bool issued = false, ok = true;
    if (a.inject) ok = warp_wait(&inject_bar, 0, wc);   // nothing arrives: runs out
    int u = 0, n = 0;
    const uint64_t kdesc = smem_desc_sw128(sbase + C::K_OFF, 16, 1024);
    const uint64_t vdesc = smem_desc_sw128(sbase + C::V_OFF, 16, 1024);
    // S^T of step uu (waits for its query/dO stage)
    auto issue_s = [&](int uu) -> bool {
      const int s = uu % kNSQ;
      if (!warp_wait(&q_full[s], (uu / kNSQ) & 1, wc)) return false;
      tc_fence_after();
      const uint64_t qd = smem_desc_sw128(sbase + C::Q_OFF + s * C::TILE, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t o = ((ks >> 2) * C::CHUNK + (ks & 3) * 32) >> 4;
        mma_ss_elect(tmem + kTST, kdesc + o, qd + o, C::ID_T, ks > 0);
      }
      issued = true;
      tc_commit_elect(&s_full);
      return true;
    };
    // dP^T of step uu (its stage already waited for by issue_s)
    auto issue_dp = [&](int uu) {
      const int s = uu % kNSQ;
      const uint64_t dd = smem_desc_sw128(sbase + C::DO_OFF + s * C::TILE, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t o = ((ks >> 2) * C::CHUNK + (ks & 3) * 32) >> 4;
        mma_ss_elect(tmem + kTDP, vdesc + o, dd + o, C::ID_T, ks > 0);
      }
      tc_commit_elect(&dp_full);
    };
    for (int it = blockIdx.x; ok && it < b.kv_total; it += gridDim.x, ++n) {
      if (!warp_wait(&kv_full, n & 1, wc)) break;
      tc_fence_after();
      if (!(ok = issue_s(u))) break;
      issue_dp(u);
      for (bool first = true;; first = false) {
        const int s = u % kNSQ;
        const int last = meta[s].last;   // read after q_full[s] (issue_s)
        const uint64_t qmn = smem_desc_sw128(sbase + C::Q_OFF + s * C::TILE, C::CHUNK, 1024);
        const uint64_t dmn = smem_desc_sw128(sbase + C::DO_OFF + s * C::TILE, C::CHUNK, 1024);
        // dV += P^T dO: packed P^T of query columns 16k..16k+15 (one K step)
        // sits in columns 16k..16k+7
        if (!warp_wait(&p_ready, u & 1, wc) || (first && n > 0 && !warp_wait(&acc_free, (n - 1) & 1, wc))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts_elect(tmem + kTDV, tmem + kTST + ks * 16, dmn + (uint64_t)(ks * 2048 >> 4), C::ID_A,
                       (!first || ks > 0) ? 1u : 0u);
        if (!last && !(ok = issue_s(u + 1))) break;
        // dK += dS^T Q
        if (!warp_wait(&ds_ready, u & 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts_elect(tmem + kTDV + D, tmem + kTDP + ks * 16, qmn + (uint64_t)(ks * 2048 >> 4), C::ID_A,
                       (!first || ks > 0) ? 1u : 0u);
        tc_commit_elect(&q_empty[s]);   // last reads of Q_u and dO_u
        if (!last) issue_dp(u + 1);
        ++u;
        if (last) break;
      }
      if (!ok) break;
      tc_commit_elect(&acc_ready);
      tc_commit_elect(&kv_empty);
    }
    if (issued) {
      tc_commit_elect(&drain_bar);
      mbar_wait_drain(&drain_bar, 0, a.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3, qd = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;                      // tile row = TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const int c0 = 32 * qd;                                 // this warp's first query column of a step
    const int gq = c0 / R;                                  // the query block of its 32 columns
    const float sl2 = a.sl2;
    constexpr int DQ = D / 4;                               // epilogue columns of dV and of dK
    int u = 0, n = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < b.kv_total; it += gridDim.x, ++n) {
      const int bh = it / b.kv_tiles, tile = it % b.kv_tiles;
      bool row_valid = false;
      int tok = 0, kk = 0, nj = 1;
      float bias = 0.f;
      if (pooled) {
        kk = tile * 128 + r;
        row_valid = kk < a.T_kv;
        if (row_valid) {
          nj = block_span(a.kept[(size_t)bh * a.T_kv + kk], a.L_src, a.L_ctx, a.b, a.T_src).y;
          bias = __log2f((float)nj);
        }
      } else {
        kk = tile * G + r / R;
        if (kk < a.T_kv) {
          const int2 sp = block_span(a.kept[(size_t)bh * a.T_kv + kk], a.L_src, a.L_ctx, a.b, a.T_src);
          nj = sp.y;
          row_valid = (r % R) < sp.y;
          tok = sp.x + r % R;
        }
      }
      for (;;) {
        const int s = u % kNSQ;
        // s_full follows q_full of the same step (the MMAs waited for it);
        // the q_full test makes the bulk-copied (lse2, Delta) visible here
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&s_full, u & 1, wc) && mbar_wait(&q_full[s], (u / kNSQ) & 1, wc))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int last = meta[s].last;
        const bool on = row_valid && ((meta[s].m[gq][r >> 5] >> (r & 31)) & 1u);
        // lse2 and Delta of this warp's 32 columns (one query block's rows
        // c0 % R .. +31), four columns per 16-byte broadcast load; rows past a
        // block's end hold (inf, 0), so P = 0 there
        const float4* dls = reinterpret_cast<const float4*>(sgen + C::DL_OFF + s * C::DL_STAGE +
                                                            (gq * 2 * R + c0 % R) * 4);
        // phase A: P^T of the 32 columns, loaded in one TMEM round trip
        float p[32];
        {
          uint32_t sv[2][16];
          tmem_ld16_pair_sync(tl + kTST + c0, sv[0], tl + kTST + c0 + 16, sv[1]);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              const float4 l4 = dls[(16 * h + e) >> 2];
              float p0 = ex2(fmaf(__uint_as_float(sv[h][e]), sl2, bias - l4.x));
              float p1 = ex2(fmaf(__uint_as_float(sv[h][e + 1]), sl2, bias - l4.y));
              float p2 = ex2(fmaf(__uint_as_float(sv[h][e + 2]), sl2, bias - l4.z));
              float p3 = ex2(fmaf(__uint_as_float(sv[h][e + 3]), sl2, bias - l4.w));
              if (!on) p0 = p1 = p2 = p3 = 0.f;
              p[16 * h + e] = p0;
              p[16 * h + e + 1] = p1;
              p[16 * h + e + 2] = p2;
              p[16 * h + e + 3] = p3;
              pk[e >> 1] = pack_bf16x2(p0, p1);
              pk[(e >> 1) + 1] = pack_bf16x2(p2, p3);
            }
            tmem_st8(tl + kTST + c0 + 16 * h, pk);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_ready);
        // phase B: dS^T = P^T (dP^T - Delta)
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&dp_full, u & 1, wc))) {
          ok = false;
          break;
        }
        tc_fence_after();
        {
          const float4* dds = dls + R / 4;   // Delta of the same columns
          uint32_t dp[2][16];
          tmem_ld16_pair_sync(tl + kTDP + c0, dp[0], tl + kTDP + c0 + 16, dp[1]);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pd[8];
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              const float4 d4 = dds[(16 * h + e) >> 2];
              const float g0 = p[16 * h + e] * (__uint_as_float(dp[h][e]) - d4.x);
              const float g1 = p[16 * h + e + 1] * (__uint_as_float(dp[h][e + 1]) - d4.y);
              const float g2 = p[16 * h + e + 2] * (__uint_as_float(dp[h][e + 2]) - d4.z);
              const float g3 = p[16 * h + e + 3] * (__uint_as_float(dp[h][e + 3]) - d4.w);
              pd[e >> 1] = pack_bf16x2(g0, g1);
              pd[(e >> 1) + 1] = pack_bf16x2(g2, g3);
            }
            tmem_st8(tl + kTDP + c0 + 16 * h, pd);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_ready);
        ++u;
        if (last) break;
      }
      if (!ok) break;
      // epilogue: this thread's DQ columns of dV and dK for tile row r
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&acc_ready, n & 1, wc))) break;
      tc_fence_after();
      // dV first, then dK, so that only one of them is held in registers
      const float sc = b.scale;
      const float inv = 1.f / (float)nj;
#pragma unroll
      for (int part = 0; part < 2; ++part) {   // 0: dV, 1: dK (scaled by s)
        uint32_t g[DQ / 16][16];
        const uint32_t col = kTDV + part * D + qd * DQ;
        __syncwarp();
        if constexpr (DQ == 32) {
          tmem_ld16_pair_sync(tl + col, g[0], tl + col + 16, g[DQ / 32]);
        } else {
          tmem_ld16_sync(tl + col, g[0]);
        }
        if (part == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_free);
        }
        if (!row_valid) continue;
        const float f = part ? sc : 1.f;
        if (pooled) {
          float4* dst = reinterpret_cast<float4*>((part ? b.dKc : b.dVc) + ((size_t)bh * a.T_kv_pad + kk) * D + qd * DQ);
#pragma unroll
          for (int e = 0; e < DQ; e += 4) {
            const uint32_t* g4 = &g[e >> 4][e & 15];
            dst[e >> 2] = make_float4(f * __uint_as_float(g4[0]), f * __uint_as_float(g4[1]),
                                      f * __uint_as_float(g4[2]), f * __uint_as_float(g4[3]));
          }
        } else {
          // this block's share of its pooled-mean gradient: dKc_j / n_j, dVc_j / n_j
          const float4* pc =
              reinterpret_cast<const float4*>((part ? b.dKc : b.dVc) + ((size_t)bh * a.T_kv_pad + kk) * D + qd * DQ);
          uint4* dst = reinterpret_cast<uint4*>((part ? b.dk : b.dv) + ((size_t)bh * a.L + tok) * D + qd * DQ);
#pragma unroll
          for (int e = 0; e < DQ; e += 8) {
            float x[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = f * __uint_as_float(g[(e + i) >> 4][(e + i) & 15]);
            if (b.has_pooled) {
              const float4 c0v = pc[e >> 2], c1v = pc[(e >> 2) + 1];
              x[0] = fmaf(c0v.x, inv, x[0]); x[1] = fmaf(c0v.y, inv, x[1]);
              x[2] = fmaf(c0v.z, inv, x[2]); x[3] = fmaf(c0v.w, inv, x[3]);
              x[4] = fmaf(c1v.x, inv, x[4]); x[5] = fmaf(c1v.y, inv, x[5]);
              x[6] = fmaf(c1v.z, inv, x[6]); x[7] = fmaf(c1v.w, inv, x[7]);
            }
            dst[e >> 3] = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                     pack_bf16x2(x[6], x[7]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// query-stationary kernel: dQ
// ---------------------------------------------------------------------------
// The forward's work items (G query blocks of one head, the same KV tiles
// and column masks).  Per tile t:
//   S = Q K_t^T, dP = dO V_t^T          (SS, M=128, N=128, K=D)
//   P = 2^(S s log2e + w - lse2), dS = P (dP - Delta)   (softmax warps, bf16 dS into TMEM)
//   dQ += dS K_t                        (TS, K_t read as the MN-major operand)
// Roles as in the forward (352 threads): warp 0 lane 0 loads Q, dO and the
// K tiles, warp 10 lane 0 the V tiles, warp 1 issues the MMAs, warps 2..9
// hold 16 query rows each (a row split between threads t and t+16).
// TMEM: S/dS buffers at 0 and 128 (tile t in t % 2), dP at 256 (one buffer,
// released as soon as the softmax warps have loaded it), dQ at 384.
constexpr int kQThreads = 352;
constexpr int kQNSK = 3;
constexpr int kQNSV = 2;
constexpr uint32_t kTS = 0;
constexpr uint32_t kTP = 256;
constexpr uint32_t kTQ = 384;

template <int D, int R>
struct QCfg {
  static constexpr int G = 128 / R;
  static constexpr int NCH = D / 64;
  static constexpr uint32_t CHUNK = 128 * 128;
  static constexpr uint32_t TILE = 128 * D * 2;
  static constexpr uint32_t BOX = R * 128;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t DO_OFF = TILE;
  static constexpr uint32_t K_OFF = 2 * TILE;
  static constexpr uint32_t V_OFF = K_OFF + kQNSK * TILE;
  static constexpr uint32_t SMEM_USED = V_OFF + kQNSV * TILE + 1024;
  static constexpr uint32_t SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, 0);
  static constexpr uint32_t ID_Q = idesc_bf16_f32(128, D, 1);
};

template <int D, int R>
__global__ void __launch_bounds__(kQThreads, 1)
    bwd_q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kp,
                 const __grid_constant__ CUtensorMap tm_vp, const __grid_constant__ CUtensorMap tm_do,
                 const BwdArgs b) {
  using C = QCfg<D, R>;
  constexpr int G = C::G;
  const AttnArgs& a = b.a;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full, q_empty, k_full[kQNSK], k_empty[kQNSK], v_full[kQNSV], v_empty[kQNSV];
  __shared__ __align__(8) uint64_t sd_full[2], dp_free, ds_full[2], dq_ready, dq_free, drain_bar, inject_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));

  if (tid == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q_empty, 1);
    for (int i = 0; i < kQNSK; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kQNSV; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sd_full[i], 1);
      mbar_init(&ds_full[i], 256);
    }
    mbar_init(&dp_free, 256);
    mbar_init(&dq_ready, 1);
    mbar_init(&dq_free, 256);
    mbar_init(&drain_bar, 1);
    mbar_init(&inject_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_kp);
    tma_prefetch_desc(&tm_vp);
  }
  if (warp == 1) tmem_alloc(&tmem_base_sh, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const WaitCtl wc{&abort_flag, a.status, a.timeout_ns};

  if ((warp == 0 || warp == 10) && lane == 0) {
    // ------------------------------------------------------------ producers
    const bool kside = warp == 0;
    int q_cnt = 0, cnt[kQNSK > kQNSV ? kQNSK : kQNSV];
    const int ns = kside ? kQNSK : kQNSV;
    for (int i = 0; i < ns; ++i) cnt[i] = 0;
    uint64_t* full = kside ? k_full : v_full;
    uint64_t* empty = kside ? k_empty : v_empty;
    const uint32_t off = kside ? C::K_OFF : C::V_OFF;
    int n = 0, t = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < a.total_items; it += gridDim.x, ++n) {
      const Item I = decode_item<G>(a, it);
      if (kside) {
        if (n >= 1 && !mbar_wait(&q_empty, (n - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(&q_full, 2 * C::TILE);
        ++q_cnt;
        for (int g = 0; g < G; ++g) {
          const int2 sp = q_span<R>(a, I, g);
          const int row = I.bh * a.L + (sp.y > 0 ? sp.x : 0);
          for (int c = 0; c < C::NCH; ++c) {
            tma_load_2d(sgen + C::Q_OFF + c * C::CHUNK + g * C::BOX, &tm_q, c * 64, row, &q_full);
            tma_load_2d(sgen + C::DO_OFF + c * C::CHUNK + g * C::BOX, &tm_do, c * 64, row, &q_full);
          }
        }
      }
      for (int j = 0; j < I.ntiles; ++j, ++t) {
        const int s = t % ns;
        if (t >= ns && !mbar_wait(&empty[s], ((t / ns) - 1) & 1, wc)) {
          ok = false;
          break;
        }
        int rows[G];
        bool pooled = false;
        for (int g = 0; g < G; ++g) {
          const int3 sp = kv_span<R, G>(a, I, j, g);
          pooled = sp.z != 0;
          rows[g] = pooled ? I.bh * a.T_kv_pad + sp.x : I.bh * a.L + (sp.y > 0 ? sp.x : 0);
        }
        const CUtensorMap* m = kside ? (pooled ? &tm_kp : &tm_k) : (pooled ? &tm_vp : &tm_v);
        mbar_arrive_expect_tx(&full[s], C::TILE);
        ++cnt[s];
        for (int g = 0; g < G; ++g)
          for (int c = 0; c < C::NCH; ++c)
            tma_load_2d(sgen + off + s * C::TILE + c * C::CHUNK + g * C::BOX, m, c * 64, rows[g], &full[s]);
      }
    }
    if (q_cnt) mbar_wait_drain(&q_full, (q_cnt - 1) & 1, a.timeout_ns);
    for (int i = 0; i < ns; ++i)
      if (cnt[i]) mbar_wait_drain(&full[i], (cnt[i] - 1) & 1, a.timeout_ns);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool issued = false, ok = true;
    if (a.inject) ok = warp_wait(&inject_bar, 0, wc);   // nothing arrives: runs out
    int n = 0, t0 = 0;
    const uint64_t qdesc = smem_desc_sw128(sbase + C::Q_OFF, 16, 1024);
    const uint64_t odesc = smem_desc_sw128(sbase + C::DO_OFF, 16, 1024);
    // S_t = Q K_t^T into buffer t % 2
    auto issue_s = [&](int t) -> bool {
      const int s = t % kQNSK;
      if (!warp_wait(&k_full[s], (t / kQNSK) & 1, wc)) return false;
      tc_fence_after();
      const uint64_t kdesc = smem_desc_sw128(sbase + C::K_OFF + s * C::TILE, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t o = ((ks >> 2) * C::CHUNK + (ks & 3) * 32) >> 4;
        mma_ss_elect(tmem + kTS + (t & 1) * 128, qdesc + o, kdesc + o, C::ID_S, ks > 0);
      }
      issued = true;
      return true;
    };
    // dP_t = dO V_t^T once the softmax warps have loaded dP_{t-1}; then S_t
    // and dP_t are announced together
    auto issue_dp = [&](int t) -> bool {
      const int s = t % kQNSV;
      if ((t > 0 && !warp_wait(&dp_free, (t - 1) & 1, wc)) || !warp_wait(&v_full[s], (t / kQNSV) & 1, wc))
        return false;
      tc_fence_after();
      const uint64_t vdesc = smem_desc_sw128(sbase + C::V_OFF + s * C::TILE, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t o = ((ks >> 2) * C::CHUNK + (ks & 3) * 32) >> 4;
        mma_ss_elect(tmem + kTP, odesc + o, vdesc + o, C::ID_S, ks > 0);
      }
      tc_commit_elect(&v_empty[s]);
      tc_commit_elect(&sd_full[t & 1]);
      return true;
    };
    for (int it = blockIdx.x; ok && it < a.total_items; it += gridDim.x, ++n) {
      const Item I = decode_item<G>(a, it);
      const int nt = I.ntiles;
      if (!warp_wait(&q_full, n & 1, wc)) break;
      tc_fence_after();
      if (!(ok = issue_s(t0) && issue_dp(t0))) break;
      if (nt == 1) tc_commit_elect(&q_empty);   // last read of this item's Q and dO
      for (int j = 0; j < nt; ++j) {
        const int t = t0 + j;
        if (j + 1 < nt) {
          if (!(ok = issue_s(t + 1) && issue_dp(t + 1))) break;
          if (j + 2 == nt) tc_commit_elect(&q_empty);
        }
        if (!warp_wait(&ds_full[t & 1], (t >> 1) & 1, wc) || (j == 0 && n > 0 && !warp_wait(&dq_free, (n - 1) & 1, wc))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t kmn = smem_desc_sw128(sbase + C::K_OFF + (t % kQNSK) * C::TILE, C::CHUNK, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts_elect(tmem + kTQ, tmem + kTS + (t & 1) * 128 + ks * 8, kmn + (uint64_t)(ks * 2048 >> 4), C::ID_Q,
                       (j > 0 || ks > 0) ? 1u : 0u);
        tc_commit_elect(&k_empty[t % kQNSK]);
      }
      if (!ok) break;
      tc_commit_elect(&dq_ready);
      t0 += nt;
    }
    if (issued) {
      tc_commit_elect(&drain_bar);
      mbar_wait_drain(&drain_bar, 0, a.timeout_ns);
    }
  } else if (warp >= 2 && warp <= 9) {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3, hw = (warp - 2) >> 2, h = lane >> 4;
    const int row = quarter * 32 + hw * 16 + (lane & 15);
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32 + hw * 16) << 16);
    const int g_r = row / R, rr = row % R;
    const float sl2 = a.sl2;
    const float log2b = __log2f((float)a.b);
    constexpr int DH = D / 2;
    int n = 0, t = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < a.total_items; it += gridDim.x, ++n) {
      const Item I = decode_item<G>(a, it);
      const int2 qs = q_span<R>(a, I, g_r);
      const bool row_valid = rr < qs.y;
      const size_t tok = (size_t)I.bh * a.L + qs.x + rr;
      const int qblk = qs.x < a.L_src ? qs.x / a.b : a.T_src + (qs.x - a.L_src) / a.b;
      const size_t dli = (((size_t)I.bh * (a.T_src + a.T_ctx) + qblk) * 2) * a.b + rr;
      const float2 mine = row_valid ? make_float2(b.dl[dli], b.dl[dli + a.b]) : make_float2(INFINITY, 0.f);
      const uint32_t* rbits = nullptr;
      int pb0 = -1, pb1 = -1;
      float d0 = 0.f, d1 = 0.f;
      if (I.kind == 2) {
        const int f = I.slot0 + g_r;
        if (f < a.n_flat) rbits = a.bits + ((size_t)I.bh * a.n_flat + f) * a.words;
        if (a.L_src % a.b) {
          pb0 = a.T_src - 1;
          d0 = (__log2f((float)(a.L_src % a.b)) - log2b) / sl2;
        }
        if ((a.L_ctx % a.b) && a.ctx_sel[(size_t)I.bh * a.K_sel + a.K_sel - 1] == a.T_ctx - 1) {
          pb1 = a.T_kv - 1;
          d1 = (__log2f((float)(a.L_ctx % a.b)) - log2b) / sl2;
        }
      }
      ItemCounts ic;
      ic.src_tail = a.L_src - (a.T_src - 1) * a.b;
      ic.kv_tail = a.b;
      if (a.ctx_sel[(size_t)I.bh * a.K_sel + a.K_sel - 1] == a.T_ctx - 1) ic.kv_tail = a.L_ctx - (a.T_ctx - 1) * a.b;
      int jm0 = -1, jm1 = -1;
      if (I.kind == 1) {
        if (ic.src_tail != a.b) jm0 = (a.T_src - 1) / G;
        jm1 = (a.T_kv - 1) / G;
      }
      int ekk = load_exact(a, I, 0, g_r);
      for (int j = 0; j < I.ntiles; ++j, ++t) {
        TileMeta cur;
        if (I.kind == 2 || j == jm0 || j == jm1) {
          cur = tile_meta<R, G>(a, I, ic, j, g_r, rbits, ekk);
          ekk = load_exact(a, I, j + 1, g_r);
        } else {
          cur.mw[0] = cur.mw[1] = cur.mw[2] = cur.mw[3] = 0xFFFFFFFFu;
          cur.pooled = 0;
          cur.masked = 0;
        }
        const int buf = t & 1;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sd_full[buf], (t >> 1) & 1, wc))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // S and dP, 32 columns of this thread's half row at a time (64
        // registers per round instead of 128)
        const float neg = (cur.pooled ? log2b : 0.f) - mine.x;
        const uint32_t wsel[2] = {h ? cur.mw[2] : cur.mw[0], h ? cur.mw[3] : cur.mw[1]};
        uint32_t pk[32];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          uint32_t sr[32], dr[32];
          tmem_ld16x2_sync2<64>(trow + kTS + buf * 128 + 32 * part, sr, trow + kTP + 32 * part, dr);
          if (part == 1) {
            tc_fence_before();
            mbar_arrive(&dp_free);   // dP of the next tile may overwrite the buffer
          }
          float s[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(sr[c]);
          if (cur.masked) {
#pragma unroll
            for (int c = 0; c < 32; ++c) s[c] = ((wsel[part] >> c) & 1u) ? s[c] : -INFINITY;
            if (cur.pooled && (pb0 >= 0 || pb1 >= 0)) {
              const int kk0 = (j - a.n_exact) * 128 + 64 * h + 32 * part;
#pragma unroll
              for (int c = 0; c < 32; ++c) s[c] += (kk0 + c == pb0) ? d0 : ((kk0 + c == pb1) ? d1 : 0.f);
            }
          }
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float p0 = ex2(fmaf(s[c], sl2, neg)), p1 = ex2(fmaf(s[c + 1], sl2, neg));
            const float g0 = p0 * (__uint_as_float(dr[c]) - mine.y);
            const float g1 = p1 * (__uint_as_float(dr[c + 1]) - mine.y);
            pk[16 * part + (c >> 1)] = pack_bf16x2(g0, g1);
          }
        }
        tmem_st16x2_32<32>(trow + kTS + buf * 128, pk);   // dS keys 64h..64h+63 -> columns 32h..32h+31
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ds_full[buf]);
      }
      if (!ok) break;
      // epilogue: dQ = s * (dS K summed over the tiles), this thread's DH columns
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&dq_ready, n & 1, wc))) break;
      tc_fence_after();
      uint32_t o[DH / 32][32];
      if constexpr (DH == 64) {
        tmem_ld16x2_sync2<DH>(trow + kTQ, o[0], trow + kTQ + 32, o[DH / 64]);
      } else {
        tmem_ld16x2_sync1<DH>(trow + kTQ, o[0]);
      }
      tc_fence_before();
      mbar_arrive(&dq_free);
      if (row_valid) {
        const float sc = b.scale;
        uint4* dst = reinterpret_cast<uint4*>(b.dq + tok * D + DH * h);
#pragma unroll
        for (int c = 0; c < DH; c += 8) {
          const uint32_t* oc = &o[c >> 5][c & 31];
          dst[c / 8] = make_uint4(pack_bf16x2(sc * __uint_as_float(oc[0]), sc * __uint_as_float(oc[1])),
                                  pack_bf16x2(sc * __uint_as_float(oc[2]), sc * __uint_as_float(oc[3])),
                                  pack_bf16x2(sc * __uint_as_float(oc[4]), sc * __uint_as_float(oc[5])),
                                  pack_bf16x2(sc * __uint_as_float(oc[6]), sc * __uint_as_float(oc[7])));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int D, int R>
static cudaError_t launch_t(const Dims& d, const CUtensorMap* maps, BwdArgs& b, int sms, cudaStream_t st) {
  using KC = KvCfg<D, R>;
  using QC = QCfg<D, R>;
  static std::atomic<unsigned long long> attr_done{0};   // per template instance
  {
    const cudaError_t e = once_per_device(attr_done, [] {
      cudaError_t r = cudaFuncSetAttribute(bwd_kv_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KC::SMEM);
      if (r == cudaSuccess)
        r = cudaFuncSetAttribute(bwd_q_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)QC::SMEM);
      return r;
    });
    if (e != cudaSuccess) return e;
  }
  const size_t entries = (size_t)d.BH * d.T * d.b;
  const int pgrid = (int)std::max<size_t>(1, std::min<size_t>((entries * (D / 8) + 255) / 256, (size_t)sms * 16));
  bwd_prep_kernel<D><<<pgrid, 256, 0, st>>>(reinterpret_cast<const uint4*>(b.o), reinterpret_cast<const uint4*>(b.dout),
                                            b.lse, b.dl, d.T, d.b, d.L, d.L_src, d.L_ctx, d.T_src, entries);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (d.K_sel < d.T_ctx) {
    bwd_zero_unkept_kernel<<<dim3(d.BH, d.T_ctx), 128, 0, st>>>(b.a.ctx_sel, d.K_sel, d.L, d.L_src, d.L_ctx, d.b, D,
                                                                 reinterpret_cast<uint4*>(b.dk),
                                                                 reinterpret_cast<uint4*>(b.dv));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (b.has_pooled) {
    b.kv_pooled = 1;
    b.kv_tiles = d.T_kv_pad / 128;
    b.kv_total = d.BH * b.kv_tiles;
    bwd_kv_kernel<D, R><<<std::min(sms, b.kv_total), kKvThreads, KC::SMEM, st>>>(maps[0], maps[1], maps[2], maps[3],
                                                                                  maps[4], maps[5], b);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  b.kv_pooled = 0;
  b.kv_tiles = (d.T_kv + KC::G - 1) / KC::G;
  b.kv_total = d.BH * b.kv_tiles;
  bwd_kv_kernel<D, R><<<std::min(sms, b.kv_total), kKvThreads, KC::SMEM, st>>>(maps[0], maps[1], maps[2], maps[3],
                                                                                maps[4], maps[5], b);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_q_kernel<D, R><<<std::min(sms, b.a.total_items), kQThreads, QC::SMEM, st>>>(maps[0], maps[1], maps[2], maps[3],
                                                                                   maps[4], maps[5], b);
  return cudaGetLastError();
}

}  // namespace bwd

cudaError_t launch_backward(const Dims& d, const CUtensorMap* maps, BwdArgs& b, int sm_count, cudaStream_t st) {
  if (d.D == 128 && d.b == 64) return bwd::launch_t<128, 64>(d, maps, b, sm_count, st);
  if (d.D == 128 && d.b == 32) return bwd::launch_t<128, 32>(d, maps, b, sm_count, st);
  if (d.D == 64 && d.b == 64) return bwd::launch_t<64, 64>(d, maps, b, sm_count, st);
  if (d.D == 64 && d.b == 32) return bwd::launch_t<64, 32>(d, maps, b, sm_count, st);
  return cudaErrorInvalidValue;
}

}  // namespace isa
