// Work items of the sparse attention kernels (forward attention and the
// query-stationary backward): which query blocks an item covers and which
// KV rows each of its 128-column tiles reads, following steps (4)-(5) of
// "Method steps in detail" on the paper.rainbus.top summary card of
// "LIVEditor-14B: Lightning Unified Video Editing via In-Context Sparse
// Attention".
//   sharp item : G = 128/R sharp blocks of one head; KV tiles run over the
//                kept blocks (source blocks, then the selected context blocks)
//   flat item  : G flat blocks of one head; first n_exact tiles whose
//                sub-block g is exact block j of query block g (block-diagonal
//                mask), then the pooled tiles: 128 rows of the head's kept
//                pooled keys/values with the row's own exact blocks masked out
//   dense item : 128 consecutive query tokens against all L tokens
#pragma once

#include "isa_common.cuh"

namespace isa {

struct Item {
  int bh, kind;     // kind: 0 dense, 1 sharp, 2 flat
  int slot0;        // first slot in the sharp/flat list, or the q tile (dense)
  int ntiles;
};

template <int G>
__device__ __forceinline__ Item decode_item(const AttnArgs& a, int it) {
  Item r;
  if (a.mode == 1) {
    r.kind = 0;
    r.bh = it / a.q_tiles;
    r.slot0 = it % a.q_tiles;
    r.ntiles = (a.L + 127) / 128;
  } else {
    // head by head: a head's sharp items, then its flat items, so the flat
    // items' exact blocks are read while the head's kept K/V is still in L2
    const int per_head = a.items_sharp + a.items_flat;
    r.bh = it / per_head;
    const int k = it % per_head;
    if (k < a.items_sharp) {
      r.kind = 1;
      r.slot0 = k * G;
      r.ntiles = (a.T_kv + G - 1) / G;
    } else {
      r.kind = 2;
      r.slot0 = (k - a.items_sharp) * G;
      r.ntiles = a.n_exact + (a.T_kv + 127) / 128;
    }
  }
  return r;
}

// (token start, valid rows) of query slot g of an item.
template <int R>
__device__ __forceinline__ int2 q_span(const AttnArgs& a, const Item& I, int g) {
  if (I.kind == 0) {
    const int s = I.slot0 * 128 + g * R;
    return make_int2(s, max(0, min(R, a.L - s)));
  }
  const int idx = I.slot0 + g;
  const int n = I.kind == 1 ? a.n_sharp : a.n_flat;
  if (idx >= n) return make_int2(0, 0);
  const int id = (I.kind == 1 ? a.sharp : a.flat)[(size_t)I.bh * n + idx];
  return block_span(id, a.L_src, a.L_ctx, a.b, a.T_src);
}

// (start row, valid rows, pooled?) of KV sub-block g of tile j.  Token rows
// are positions in [0, L); pooled rows are positions in the head's Kp/Vp.
template <int R, int G>
__device__ __forceinline__ int3 kv_span(const AttnArgs& a, const Item& I, int j, int g) {
  if (I.kind == 0) {
    const int s = j * 128 + g * R;
    return make_int3(s, max(0, min(R, a.L - s)), 0);
  }
  if (I.kind == 1) {
    const int kk = j * G + g;
    if (kk >= a.T_kv) return make_int3(0, 0, 0);
    const int2 sp = block_span(a.kept[(size_t)I.bh * a.T_kv + kk], a.L_src, a.L_ctx, a.b, a.T_src);
    return make_int3(sp.x, sp.y, 0);
  }
  if (j < a.n_exact) {
    const int f = I.slot0 + g;
    if (f >= a.n_flat) return make_int3(0, 0, 0);
    const int kk = a.exact[((size_t)I.bh * a.n_flat + f) * a.n_exact + j];
    const int2 sp = block_span(a.kept[(size_t)I.bh * a.T_kv + kk], a.L_src, a.L_ctx, a.b, a.T_src);
    return make_int3(sp.x, sp.y, 0);
  }
  const int r0 = (j - a.n_exact) * 128 + g * R;
  return make_int3(r0, max(0, min(R, a.T_kv - r0)), 1);
}

// Per-item constants that give the valid-token count of any kept block
// without a memory access: only the last source block and the last context
// block can be partial, and the latter is kept only as the last kept block.
struct ItemCounts {
  int src_tail;     // tokens of block T_src-1
  int kv_tail;      // tokens of kept block T_kv-1
};

__device__ __forceinline__ int kept_count(const AttnArgs& a, const ItemCounts& ic, int kk) {
  if (kk >= a.T_kv || kk < 0) return 0;
  if (kk == a.T_src - 1) return ic.src_tail;
  if (kk == a.T_kv - 1) return ic.kv_tail;
  return a.b;
}

// Column validity of one KV tile for one query row: bit c of mw[c/32] set
// when column c takes part.  `masked` is warp-uniform (a row-independent
// mask for sharp and dense tiles; flat tiles are always masked).
struct TileMeta {
  uint32_t mw[4];
  int pooled, masked;
};

// exact-block position (in the kept list) of query block g_r of a flat item
// for exact tile j (-1 outside the exact tiles): loaded one tile ahead of its
// use; a row needs only its own query block's entry
__device__ __forceinline__ int load_exact(const AttnArgs& a, const Item& I, int j, int g_r) {
  const int f = I.slot0 + g_r;
  return (I.kind == 2 && j < a.n_exact && f < a.n_flat) ? a.exact[((size_t)I.bh * a.n_flat + f) * a.n_exact + j] : -1;
}

template <int R, int G>
__device__ __forceinline__ TileMeta tile_meta(const AttnArgs& a, const Item& I, const ItemCounts& ic, int j, int g_r,
                                              const uint32_t* rbits, int ekk_r) {
  TileMeta m;
  if (I.kind == 2 && j >= a.n_exact) {
    // pooled tile: kept blocks [jp*128, jp*128+128) minus this row's exact blocks
    const int jp = j - a.n_exact;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int rem = a.T_kv - (jp * 128 + 32 * w);
      const uint32_t range = rem >= 32 ? 0xFFFFFFFFu : (rem <= 0 ? 0u : ((1u << rem) - 1u));
      const int wi = jp * 4 + w;
      const uint32_t ex = rbits ? (wi < a.words ? rbits[wi] : 0u) : 0xFFFFFFFFu;
      m.mw[w] = range & ~ex;
    }
    m.pooled = 1;
    m.masked = 1;
    return m;
  }
  int cnt[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (I.kind == 0) {
      const int s0 = j * 128 + g * R;
      cnt[g] = max(0, min(R, a.L - s0));
    } else if (I.kind == 1) {
      cnt[g] = kept_count(a, ic, j * G + g);
    } else {
      cnt[g] = (g == g_r) ? kept_count(a, ic, ekk_r) : 0;   // block-diagonal exact tiles
    }
  }
  bool full = true;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int c = cnt[(w * 32) / R] - (w * 32) % R;
    m.mw[w] = c >= 32 ? 0xFFFFFFFFu : (c <= 0 ? 0u : ((1u << c) - 1u));
    full = full && m.mw[w] == 0xFFFFFFFFu;
  }
  m.pooled = 0;
  m.masked = (I.kind == 2) ? 1 : (full ? 0 : 1);
  return m;
}

// TMEM loads of 16 lanes with the columns split between the two half warps
// (the .16x32bx2 shape): thread t < 16 reaches lane base+t, columns
// [c, c+32); thread t >= 16 reaches lane base+t-16, columns [c+SPLIT,
// c+SPLIT+32).  So both 64-column halves of a row sit in one warp.  Each
// helper issues its groups and their tcgen05.wait::ld in one asm statement
// (see tmem_ld16_pair_sync).  One group:
template <int SPLIT>
__device__ __forceinline__ void tmem_ld16x2_sync1(uint32_t t0, uint32_t (&r0)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], %33;\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ISA_R32(r0)
      : "r"(t0), "n"(SPLIT)
      : "memory");
}
// One 16-column group (thread t < 16: columns [c, c+16), t >= 16:
// [c+SPLIT, c+SPLIT+16)) and the wait:
template <int SPLIT>
__device__ __forceinline__ void tmem_ld16x2_sync1_16(uint32_t t0, uint32_t (&r0)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], %17;\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ISA_R16(r0)
      : "r"(t0), "n"(SPLIT)
      : "memory");
}
// Two groups and the wait:
template <int SPLIT>
__device__ __forceinline__ void tmem_ld16x2_sync2(uint32_t t0, uint32_t (&r0)[32], uint32_t t1, uint32_t (&r1)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64], %66;\n\t"
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65], %66;\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ISA_R32(r0), ISA_R32(r1)
      : "r"(t0), "r"(t1), "n"(SPLIT)
      : "memory");
}
// Four groups and the wait:
template <int SPLIT>
__device__ __forceinline__ void tmem_ld16x2_sync4(uint32_t t0, uint32_t (&r0)[32], uint32_t t1, uint32_t (&r1)[32],
                                                  uint32_t t2, uint32_t (&r2)[32], uint32_t t3, uint32_t (&r3)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%128], %132;\n\t"
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%129], %132;\n\t"
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95}, [%130], %132;\n\t"
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,"
      "%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%131],"
      " %132;\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : ISA_R32(r0), ISA_R32(r1), ISA_R32(r2), ISA_R32(r3)
      : "r"(t0), "r"(t1), "r"(t2), "r"(t3), "n"(SPLIT)
      : "memory");
}
// Stores of 16 and 8 columns in the same split layout.
template <int SPLIT>
__device__ __forceinline__ void tmem_st16x2_16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], %1, {%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17};" ::
          "r"(taddr),
      "n"(SPLIT), ISA_W16(r)
      : "memory");
}
template <int SPLIT>
__device__ __forceinline__ void tmem_st16x2_8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.16x32bx2.x8.b32 [%0], %1, {%2,%3,%4,%5,%6,%7,%8,%9};" ::"r"(taddr), "n"(SPLIT),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
template <int SPLIT>
__device__ __forceinline__ void tmem_st16x2_32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], %1, {%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%"
      "17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33};" ::"r"(taddr),
      "n"(SPLIT), ISA_W32(r)
      : "memory");
}

// Warp-uniform bounded wait: every lane waits, the warp agrees on the result.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, w));
}

}  // namespace isa
