// Attention kernel of the ISA forward pass for sm_100a: steps (4)-(6) of
// "Method steps in detail" on the paper.rainbus.top summary card of
// "LIVEditor-14B: Lightning Unified Video Editing via In-Context Sparse
// Attention", with the 0th-order Taylor term of its "0th-order Taylor
// approximate attention" section, and the dense attention it replaces.
//
// One persistent launch walks a list of work items.  An item is a 128-row
// query tile made of G = 128/R query blocks of R = b rows and a sequence of
// 128-column KV tiles, each made of G sub-blocks of R rows:
//   sharp item : G sharp blocks of one head; KV tiles run over the kept
//                blocks (source blocks, then the selected context blocks)
//   flat item  : G flat blocks of one head; first n_exact tiles whose
//                sub-block g is exact block j of query block g (block-diagonal:
//                a softmax warp's rows, one query block, load and exponentiate
//                only their own sub-block's columns and write zeros for the
//                rest of P), then the pooled tiles: 128 rows of the head's kept
//                pooled keys/values (Kp, Vp) with logit bias log2(n_j) and the
//                row's own exact blocks masked out
//   dense item : 128 consecutive query tokens against all L tokens
// All tiles of an item update one online-softmax state per query row, so the
// exact and the pooled terms share one normaliser.
//
// Roles (352 threads, one CTA per SM):
//   warp 0 lane 0 : TMA producer of the Q tile and the K tiles (kNSK stages)
//   warp 1        : allocates TMEM; runs the MMA loop as one converged warp,
//                   one elected lane issuing each tcgen05.mma / commit
//   warps 2..9    : softmax / correction / epilogue; each warp owns 16 query
//                   rows, each row split between threads t and t+16 of the
//                   warp (64 columns of the S tile each)
//   warp 10 lane 0: TMA producer of the V tiles (kNSV stages)
// TMEM (512 columns): S0 [0,128), S1 [128,256), S2 [256,384), O [384, 384+D).
// S of tile t lives in buffer t % 3, so S runs two tiles ahead of P.V.  P (bf16)
// overwrites the first 64 columns of its S buffer and feeds the P.V MMA as the
// A operand straight from TMEM.
#include "isa_common.cuh"
#include "isa_items.cuh"

namespace isa {

constexpr int kThreads = 352;      // 11 warps: Q/K producer, MMA, 8 softmax, V producer
constexpr int kNSK = 3;             // K pipeline stages
constexpr int kNSV = 2;             // V pipeline stages
constexpr float kRescaleLog2 = 8.f; // lazy rescaling threshold (log2 units)
constexpr uint32_t kTmemO = 384;    // TMEM column of O (after three 128-column S buffers)

template <bool B>
struct FlatTag {
  static constexpr bool value = B;
};

template <int D, int R>
struct Cfg {
  static constexpr int G = 128 / R;
  static constexpr int NCH = D / 64;                       // 64-column chunks of a row
  static constexpr uint32_t CHUNK = 128 * 128;             // 128 rows x 128 bytes
  static constexpr uint32_t TILE = 128 * D * 2;            // one 128-row tile
  static constexpr uint32_t BOX = R * 128;                 // one TMA box
  static constexpr uint32_t Q_OFF = 0;                     // one Q tile
  static constexpr uint32_t K_OFF = TILE;
  static constexpr uint32_t V_OFF = K_OFF + kNSK * TILE;
  // + 1024 alignment slack; at least 120 KB so that only one CTA (and one
  // 512-column TMEM allocation) fits on an SM
  static constexpr uint32_t SMEM_USED = V_OFF + kNSV * TILE + 1024;
  static constexpr uint32_t SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, 0);
  static constexpr uint32_t ID_O = idesc_bf16_f32(128, D, 1);
};

template <int D, int R>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kp,
                const __grid_constant__ CUtensorMap tm_vp, const AttnArgs a) {
  using C = Cfg<D, R>;
  constexpr int G = C::G;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full, q_empty, k_full[kNSK], k_empty[kNSK], v_full[kNSV], v_empty[kNSV];
  __shared__ __align__(8) uint64_t s_full[3], p_full[3], pv_done[2], o_ready, o_free, drain_bar, inject_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));

  if (tid == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q_empty, 1);
    for (int i = 0; i < 3; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 256);
    }
    for (int i = 0; i < kNSK; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kNSV; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(&o_ready, 1);
    mbar_init(&o_free, 256);
    mbar_init(&drain_bar, 1);
    mbar_init(&inject_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
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
    // warp 0: Q tile and K tiles; warp 10: V tiles.  Separate threads keep
    // the K stream kNSK tiles and the V stream kNSV tiles ahead of the MMA
    // independently of each other.
    const bool kside = warp == 0;
    int q_cnt = 0, cnt[kNSK > kNSV ? kNSK : kNSV];
    const int ns = kside ? kNSK : kNSV;
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
        mbar_arrive_expect_tx(&q_full, C::TILE);
        ++q_cnt;
        for (int g = 0; g < G; ++g) {
          const int2 sp = q_span<R>(a, I, g);
          const int row = I.bh * a.L + (sp.y > 0 ? sp.x : 0);
          for (int c = 0; c < C::NCH; ++c)
            tma_load_2d(sgen + C::Q_OFF + c * C::CHUNK + g * C::BOX, &tm_q, c * 64, row, &q_full);
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
    // let every copy in flight land before the CTA can exit
    if (q_cnt) mbar_wait_drain(&q_full, (q_cnt - 1) & 1, a.timeout_ns);
    for (int i = 0; i < ns; ++i)
      if (cnt[i]) mbar_wait_drain(&full[i], (cnt[i] - 1) & 1, a.timeout_ns);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop in lockstep, so every descriptor and TMEM
    // address is warp-uniform; one elected lane issues each tcgen05 op.  S of
    // tile t+2 is issued before P.V of tile t (three S buffers), so the
    // softmax of the next two tiles never waits for the P.V round trip.
    bool issued = false, ok = true;
    if (a.inject) ok = warp_wait(&inject_bar, 0, wc);   // nothing arrives: runs out
    int n = 0, t0 = 0;   // items so far, global index of the item's first tile
    const uint32_t tO = tmem + kTmemO;
    // Descriptors are built once per operand tile; the per-K-step offsets are
    // added to the start-address field (address / 16, 14 bits: shared memory
    // is below 256 KB, so the addition never carries out of the field).
    const uint64_t qdesc = smem_desc_sw128(sbase + C::Q_OFF, 16, 1024);
    // S_t = Q K_t^T into S buffer t % 3 (k_ready: K_t is known to have landed)
    auto issue_s = [&](int t, bool last, bool k_ready) -> bool {
      const int s = t % kNSK;
      if (!k_ready && !warp_wait(&k_full[s], (t / kNSK) & 1, wc)) return false;
      tc_fence_after();
      const uint64_t kdesc = smem_desc_sw128(sbase + C::K_OFF + s * C::TILE, 16, 1024);
      const uint32_t tS = tmem + (t % 3) * 128;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t o = ((ks >> 2) * C::CHUNK + (ks & 3) * 32) >> 4;
        mma_ss_elect(tS, qdesc + o, kdesc + o, C::ID_S, ks > 0);
      }
      issued = true;
      tc_commit_elect(&s_full[t % 3]);
      tc_commit_elect(&k_empty[s]);
      if (last) tc_commit_elect(&q_empty);   // last read of this item's Q
      return true;
    };
    for (int it = blockIdx.x; ok && it < a.total_items; it += gridDim.x, ++n) {
      const Item I = decode_item<G>(a, it);
      const int nt = I.ntiles;
      if (!warp_wait(&q_full, n & 1, wc)) break;
      tc_fence_after();
      for (int j = 0; ok && j < nt && j < 2; ++j) ok = issue_s(t0 + j, j == nt - 1, false);
      for (int j = 0; ok && j < nt; ++j) {
        const int tp = t0 + j, sp = tp % kNSV, pb = tp % 3, ts = tp + 2;
        const bool do_s = j + 2 < nt, first_pv = j == 0 && n > 0;
        // Test everything this step needs at once, without blocking: the
        // tests' latencies overlap, and the MMA queue is shallow, so a chain
        // of waits here would leave the tensor pipe idle.  Blocking waits
        // remain only for what is not ready yet.
        uint32_t r = (do_s ? (uint32_t)mbar_test(&k_full[ts % kNSK], (ts / kNSK) & 1) : 1u) |
                     ((uint32_t)mbar_test(&p_full[pb], (tp / 3) & 1) << 1) |
                     ((uint32_t)mbar_test(&v_full[sp], (tp / kNSV) & 1) << 2) |
                     ((first_pv ? (uint32_t)mbar_test(&o_free, (n - 1) & 1) : 1u) << 3);
        r = __reduce_and_sync(0xFFFFFFFFu, r);
        if (do_s && !(ok = issue_s(ts, ts == t0 + nt - 1, (r & 1u) != 0))) break;
        // O (+)= P_tp V_tp
        if ((!(r & 2u) && !warp_wait(&p_full[pb], (tp / 3) & 1, wc)) ||
            (!(r & 4u) && !warp_wait(&v_full[sp], (tp / kNSV) & 1, wc)) ||
            (!(r & 8u) && !warp_wait(&o_free, (n - 1) & 1, wc))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t vdesc = smem_desc_sw128(sbase + C::V_OFF + sp * C::TILE, C::CHUNK, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts_elect(tO, tmem + pb * 128 + ks * 8, vdesc + (uint64_t)(ks * 2048 >> 4), C::ID_O,
                       (j > 0 || ks > 0) ? 1u : 0u);
        tc_commit_elect(&v_empty[sp]);
        tc_commit_elect(&pv_done[tp & 1]);
      }
      if (!ok) break;
      tc_commit_elect(&o_ready);   // once per item: every P.V of the item landed in O
      t0 += nt;
    }
    if (issued) {
      tc_commit_elect(&drain_bar);
      mbar_wait_drain(&drain_bar, 0, a.timeout_ns);
    }
  } else if (warp >= 2 && warp <= 9) {
    // ------------------------------------------------------------ softmax
    // Warps 2..9.  Two warps share each TMEM lane quarter (tcgen05 access
    // reaches lanes 32*(warp%4)..+31): warp half hw takes lanes 16*hw..+15 of
    // the quarter, i.e. 16 query rows.  Thread t < 16 holds columns 0..63 of
    // row t of the group (h = 0), thread t+16 columns 64..127 of the same row
    // (h = 1): the row maximum is one shuffle, the two partial normalisers are
    // added in the epilogue, and the two warps never wait for each other.
    const int quarter = warp & 3, hw = (warp - 2) >> 2, h = lane >> 4;
    const int row = quarter * 32 + hw * 16 + (lane & 15);
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32 + hw * 16) << 16);   // first lane of the group
    const int g_r = row / R, rr = row % R;
    const float sl2 = a.sl2;
    const float log2b = __log2f((float)a.b);
    constexpr int DH = D / 2;           // output columns of this half
    int n = 0, t = 0;
    bool ok = true, s_ready = false;   // s_ready: S of tile t known complete
    for (int it = blockIdx.x; ok && it < a.total_items; it += gridDim.x, ++n) {
      const Item I = decode_item<G>(a, it);
      const int2 qs = q_span<R>(a, I, g_r);
      const bool row_valid = rr < qs.y;
      // pooled tiles of a flat item: this row's exact-block bitmap and the
      // (at most two) partial kept blocks, whose weight is n_j instead of b
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
      if (I.kind != 0 && a.ctx_sel[(size_t)I.bh * a.K_sel + a.K_sel - 1] == a.T_ctx - 1)
        ic.kv_tail = a.L_ctx - (a.T_ctx - 1) * a.b;
      float m_run = -INFINITY, l_run = 0.f;
      int jm0 = -1, jm1 = -1;
      if (I.kind == 1) {
        if (ic.src_tail != a.b) jm0 = (a.T_src - 1) / G;
        jm1 = (a.T_kv - 1) / G;
      } else if (I.kind == 0) {
        jm1 = (a.L - 1) / 128;
      }
      int ekk = load_exact(a, I, 0, g_r);
      // Two instances of the tile loop: flat items (with the block-diagonal
      // exact tiles) and the rest, so the hot loop of sharp items carries no
      // code of the other.
      auto tile_loop = [&](auto flat_tag) {
        constexpr bool FLAT = decltype(flat_tag)::value;
        for (int j = 0; j < I.ntiles; ++j, ++t) {
          // An exact tile of a flat item is block-diagonal: this warp's rows
          // (one query block) take part only in the columns of their own
          // sub-block, [g_r*R, g_r*R + dcnt).  Only those columns are loaded
          // and exponentiated; P is zero elsewhere.
          const bool diag = FLAT && j < a.n_exact;   // warp-uniform
          int dcnt = R;
          TileMeta cur;
          if (diag) {
            dcnt = kept_count(a, ic, ekk);
            ekk = load_exact(a, I, j + 1, g_r);
          } else if (FLAT || j == jm0 || j == jm1) {
            cur = tile_meta<R, G>(a, I, ic, j, g_r, rbits, ekk);
            ekk = load_exact(a, I, j + 1, g_r);
          } else {
            cur.mw[0] = cur.mw[1] = cur.mw[2] = cur.mw[3] = 0xFFFFFFFFu;
            cur.pooled = 0;
            cur.masked = 0;
          }
          const int buf = t % 3;
          if (!s_ready && !__all_sync(0xFFFFFFFFu, mbar_wait(&s_full[buf], (t / 3) & 1, wc))) {
            ok = false;
            break;
          }
          tc_fence_after();
          bool need, s_next;
          float alpha;
          if (diag) {
            constexpr int NC = R / 2;   // columns per thread: half of the row's own sub-block
            uint32_t sr[NC];
            if constexpr (NC == 32) {
              tmem_ld16x2_sync1<32>(trow + buf * 128 + g_r * R, sr);
            } else {
              tmem_ld16x2_sync1_16<16>(trow + buf * 128 + g_r * R, sr);
            }
            float s[NC];
#pragma unroll
            for (int c = 0; c < NC; ++c) s[c] = __uint_as_float(sr[c]);
            if (dcnt < R) {
#pragma unroll
              for (int c = 0; c < NC; ++c) s[c] = (h * NC + c < dcnt) ? s[c] : -INFINITY;
            }
            float mxa[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mxa[e] = -INFINITY;
#pragma unroll
            for (int c = 0; c < NC; c += 2) mxa[(c >> 1) & 7] = fmax3(mxa[(c >> 1) & 7], s[c], s[c + 1]);
            const float mh = fmax3(fmax3(mxa[0], mxa[1], mxa[2]), fmax3(mxa[3], mxa[4], mxa[5]), fmaxf(mxa[6], mxa[7]));
            const float mx = fmaxf(mh, __shfl_xor_sync(0xFFFFFFFFu, mh, 16)) * sl2;   // whole row
            need = mx > m_run + kRescaleLog2;
            const float m_new = need ? mx : m_run;
            const float m_ref = (m_new == -INFINITY) ? 0.f : m_new;
            alpha = need ? ex2(m_run - m_ref) : 1.f;
            const float neg = -m_ref;
            s_next = mbar_test(&s_full[(t + 1) % 3], ((t + 1) / 3) & 1);
            float2 acc[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[e] = make_float2(0.f, 0.f);
            uint32_t pk[NC / 2];
#pragma unroll
            for (int c = 0; c < NC; c += 2) {
              const float2 x = ffma2(make_float2(s[c], s[c + 1]), make_float2(sl2, sl2), make_float2(neg, neg));
              const float2 pp = make_float2(ex2(x.x), ex2(x.y));   // MUFU: 2^-inf is +0 for masked columns
              acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], pp);
              pk[c >> 1] = pack_bf16x2(pp.x, pp.y);
            }
            const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
            const float2 a03 = fadd2(a01, a23);
            l_run = l_run * alpha + (a03.x + a03.y);
            m_run = m_new;
            // P keys g_r*R + h*NC .. +NC-1 -> columns g_r*R/2 + h*NC/2 ..; zeros
            // in the other sub-blocks' columns
            const uint32_t zero[NC / 2] = {};
            if constexpr (NC == 32) {
              tmem_st16x2_16<16>(trow + buf * 128 + 32 * g_r, pk);
              tmem_st16x2_16<16>(trow + buf * 128 + 32 * (1 - g_r), zero);
            } else {
              tmem_st16x2_8<8>(trow + buf * 128 + 16 * g_r, pk);
#pragma unroll
              for (int g2 = 1; g2 < 4; ++g2) tmem_st16x2_8<8>(trow + buf * 128 + 16 * ((g_r + g2) & 3), zero);
            }
          } else {
            uint32_t sr[2][32];
            // columns 64h + 0..31 and 64h + 32..63, waited for in the same statement
            tmem_ld16x2_sync2<64>(trow + buf * 128, sr[0], trow + buf * 128 + 32, sr[1]);
            float s[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);
            if (cur.masked) {
              const uint32_t w0 = h ? cur.mw[2] : cur.mw[0], w1 = h ? cur.mw[3] : cur.mw[1];
#pragma unroll
              for (int c = 0; c < 64; ++c) s[c] = ((((c < 32) ? w0 : w1) >> (c & 31)) & 1u) ? s[c] : -INFINITY;
              if (cur.pooled && (pb0 >= 0 || pb1 >= 0)) {
                const int kk0 = (j - a.n_exact) * 128 + 64 * h;
#pragma unroll
                for (int c = 0; c < 64; ++c) s[c] += (kk0 + c == pb0) ? d0 : ((kk0 + c == pb1) ? d1 : 0.f);
              }
            }
            // half-row maximum: 8 independent chains of 3-input max
            float mxa[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mxa[e] = -INFINITY;
#pragma unroll
            for (int c = 0; c < 64; c += 2) mxa[(c >> 1) & 7] = fmax3(mxa[(c >> 1) & 7], s[c], s[c + 1]);
            const float mh = fmax3(fmax3(mxa[0], mxa[1], mxa[2]), fmax3(mxa[3], mxa[4], mxa[5]), fmaxf(mxa[6], mxa[7]));
            const float bias = cur.pooled ? log2b : 0.f;
            const float mx = fmaxf(mh, __shfl_xor_sync(0xFFFFFFFFu, mh, 16)) * sl2 + bias;   // whole row
            need = mx > m_run + kRescaleLog2;
            const float m_new = need ? mx : m_run;
            const float m_ref = (m_new == -INFINITY) ? 0.f : m_new;
            alpha = need ? ex2(m_run - m_ref) : 1.f;
            const float neg = bias - m_ref;
            // Is S of the next tile (t+1, possibly the next item's first) there
            // already?  The test's latency overlaps the exponentials below, and a
            // set phase stays set until the softmax has consumed that tile.
            s_next = mbar_test(&s_full[(t + 1) % 3], ((t + 1) / 3) & 1);
            // p = 2^(s * scale*log2e + bias - m_ref) in pairs; bf16 P for the MMA
            float2 acc[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[e] = make_float2(0.f, 0.f);
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const float2 x = ffma2(make_float2(s[c], s[c + 1]), make_float2(sl2, sl2), make_float2(neg, neg));
              const float2 pp = make_float2(ex2(x.x), ex2(x.y));   // MUFU; 2^-inf = +0 for masked columns
              acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], pp);
              pk[c >> 1] = pack_bf16x2(pp.x, pp.y);
            }
            const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
            const float2 a03 = fadd2(a01, a23);
            l_run = l_run * alpha + (a03.x + a03.y);
            m_run = m_new;
            tmem_st16x2_32<32>(trow + buf * 128, pk);   // P keys 64h..64h+63 -> columns 32h..32h+31
          }
          if (j > 0 && __any_sync(0xFFFFFFFFu, need)) {
            // rescale this half of the running output once P.V of the previous
            // tile landed.  pv_done[u & 1] completes once per P.V of tile u, so
            // P.V t-1 is phase (t-1)>>1 of pv_done[(t-1) & 1]; the phase before
            // it (P.V t-3) has completed because S_t, ready here, was issued
            // after P.V t-3, so the parity test is exact.
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&pv_done[(t - 1) & 1], ((t - 1) >> 1) & 1, wc))) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < DH; c0 += 32) {
              uint32_t o[32];
              tmem_ld16x2_sync1<DH>(trow + kTmemO + c0, o);   // columns DH*h + c0..+31
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st16x2_32<DH>(trow + kTmemO + c0, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&p_full[buf]);
          s_ready = __all_sync(0xFFFFFFFFu, s_next);
        }
      };
      if (I.kind == 2) tile_loop(FlatTag<true>{}); else tile_loop(FlatTag<false>{});
      if (!ok) break;
      // epilogue: wait until every P.V of the item landed (a per-item barrier:
      // pv_done may still be two phases behind here, because the last tile's
      // S MMA was issued before the second-to-last P.V), add the partial
      // normalisers of the row's two threads, normalise and write this
      // thread's DH output columns of the row
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&o_ready, n & 1, wc))) break;
      tc_fence_after();
      uint32_t o[DH / 32][32];
      if constexpr (DH == 64) {
        tmem_ld16x2_sync2<DH>(trow + kTmemO, o[0], trow + kTmemO + 32, o[DH / 64]);
      } else {
        tmem_ld16x2_sync1<DH>(trow + kTmemO, o[0]);
      }
      tc_fence_before();
      mbar_arrive(&o_free);
      const float l_tot = l_run + __shfl_xor_sync(0xFFFFFFFFu, l_run, 16);
      if (row_valid) {
        const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
        const size_t tok = (size_t)I.bh * a.L + qs.x + rr;
        uint4* dst = reinterpret_cast<uint4*>(a.out + tok * D + DH * h);
#pragma unroll
        for (int c = 0; c < DH; c += 8) {
          uint4 w;
          const uint32_t* oc = &o[c >> 5][c & 31];
          w.x = pack_bf16x2(__uint_as_float(oc[0]) * inv, __uint_as_float(oc[1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(oc[2]) * inv, __uint_as_float(oc[3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(oc[4]) * inv, __uint_as_float(oc[5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(oc[6]) * inv, __uint_as_float(oc[7]) * inv);
          dst[c / 8] = w;
        }
        if (a.lse && h == 0) {
          const float mref = m_run == -INFINITY ? 0.f : m_run;
          a.lse[tok] = (mref + __log2f(l_tot)) * 0.69314718055994531f;
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
static cudaError_t launch_t(const CUtensorMap* maps, const AttnArgs& a, int grid, cudaStream_t st) {
  using C = Cfg<D, R>;
  static std::atomic<unsigned long long> attr_done{0};   // per template instance
  cudaError_t e = once_per_device(attr_done, [] {
    return cudaFuncSetAttribute(attn_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  });
  if (e != cudaSuccess) return e;
  attn_kernel<D, R><<<grid, kThreads, C::SMEM, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], a);
  return cudaGetLastError();
}

cudaError_t launch_attention(int D, int R, const CUtensorMap* maps, const AttnArgs& a, int grid, cudaStream_t st) {
  if (D == 128 && R == 64) return launch_t<128, 64>(maps, a, grid, st);
  if (D == 128 && R == 32) return launch_t<128, 32>(maps, a, grid, st);
  if (D == 64 && R == 64) return launch_t<64, 64>(maps, a, grid, st);
  if (D == 64 && R == 32) return launch_t<64, 32>(maps, a, grid, st);
  return cudaErrorInvalidValue;
}

}  // namespace isa
