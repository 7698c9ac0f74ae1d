// fwd_sm100.cuh — persistent, warp-specialised forward kernel of exact attention for sm_100a.
//
// Computes, for every (segment, query-tile pair, head block), out = softmax(QK^T*scale+bias)V
// and lse, one 128-key tile at a time with an online softmax, so the score matrix only ever
// lives in tensor memory (the blockwise engine of "大模型推理加速终极指南", section 1; masks and
// bias of "How to Build Memory-Efficient Transformers with xFormers…", techniques 1, 3 and 5).
//
// A work item is a pair of 128-row query sub-tiles (h = 0, 1) that share every K/V tile.
// Roles (384 threads, one CTA per SM; warps 10-11 only lend their registers):
//   warps 0-3  softmax / correction / epilogue of sub-tile 0: thread r owns row r = TMEM lane r.
//   warps 4-7  the same for sub-tile 1.
//   warp 8     tcgen05 issuer (one lane); also allocates TMEM. Per K/V tile j it issues
//              PV_0(j-1), QK_0(j), PV_1(j-1), QK_1(j): while one warpgroup turns S_h(j) into
//              P_h(j), the tensor core works on the other sub-tile, and when S_h(j) is ready the
//              earlier PV_h(j-1) has completed, so O_h can be rescaled without another wait.
//   warp 9     scheduler and TMA producer: walks this CTA's work items, hands each one, decoded,
//              to the other roles through a small queue in shared memory, then loads both Q
//              sub-tiles of the item and streams K_j, V_j through an NS-slot ring.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256, 256+D), O_1 [256+D, 256+2D). P_h(j) is
// written bf16/f16-packed over the first 64 columns of S_h and read from there as the A operand.
//
// GQA packing: a 128-row sub-tile holds 128/P tokens x P query heads of one KV group (row r ->
// token tok0 + h*128/P + r/P, head hb*P + r%P), loaded by one 3-D TMA box [128/P tokens, P heads,
// 64 d], so each K/V tile is read once for the 2P heads/2*128/P tokens that share it.
//
// Schedule: only live items are visited. Segments are ranked by their number of query-tile pairs
// at CTA start; items are ordered level by level (pair index from the last, i.e. heaviest first
// for causal masks), and within a level by segment rank and head block, so the segments live at a
// level form a prefix of the ranking. CTA b of G takes items b, 2G-1-b, 2G+b, 4G-1-b, ...
// (a zig-zag over the heavy-first list), which balances the persistent CTAs without any counter
// in global memory, so concurrent launches stay independent.
//
// Epilogue: each softmax warp stages its 32 output rows in shared memory (128-byte swizzle) and
// writes them with TMA stores, one 64-column box at a time; rows of a segment's partial last tile
// are written by plain stores so that nothing past the segment is touched.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <type_traits>

#include "ptx.cuh"

namespace mea {

struct FwdParams {
  void* out;
  float* lse;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const float* slopes;
  int n_seqs;
  int total_q;
  int hq;
  int dh;            // head dim of q, k, v and out rows (<= D; the TMA zero-fills columns past it)
  int n_hb;          // head blocks = hq / P
  int P;             // query heads packed per sub-tile (a power of two dividing R)
  int R;             // query heads per KV head
  int tok_per_tile;  // 128 / P tokens per sub-tile
  int subtiles;      // query sub-tiles per work item (2; 1 for the 256-wide kernel)
  // P and subtiles * tok_per_tile (tokens per item) are powers of two; the KV group of head
  // block hb is (hb * g_mul) >> 32 with g_mul = ceil(2^32 / (R / P)) (exact for hb * (R / P) <
  // 2^32).
  int log2_p;
  int log2_tpp;
  unsigned long long g_mul;
  float c1;          // scale * log2(e) (times the q and k descales for 8-bit inputs)
  float o_scale;     // multiplies O before the division by l (the v descale; 1 for 16-bit)
  unsigned long long timeout_ns;
};

// E8: q, k, v are 8-bit e4m3 (kind::f8f6f4 MMAs, P handed over as e4m3); otherwise 16-bit.
template <int D, bool E8 = false>
struct FwdCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int ELEM = E8 ? 1 : 2;                // bytes per q/k/v element
  static constexpr int ATOM_COLS = 128 / ELEM;           // elements per 128-byte swizzle row
  static constexpr int ATOMS = D / ATOM_COLS;            // 128-byte swizzle atoms along D
  static constexpr int KSTEP = 32 / ELEM;                // K elements per MMA (32 bytes)
  static constexpr int P_COLS = 128 * ELEM / 4;          // TMEM columns holding P of one tile
  static constexpr uint32_t ATOM_BYTES = 128 * 128;
  static constexpr uint32_t TILE_BYTES = 128 * D * ELEM;
  static constexpr int NS = E8 ? 10 : ((D == 128) ? 4 : 8);
  static constexpr int OUT_ATOMS = D / 64;               // 128-byte atoms of a 16-bit out row
  static constexpr uint32_t STG_WARP = 32 * 128;         // one warp's 32 rows x one out atom
  static constexpr int QD = 4;                           // work-item queue depth
  static constexpr int MAXSEG = 256;                     // segments ranked in shared memory
  static constexpr uint32_t SMEM_Q = 0;                  // two Q sub-tiles
  static constexpr uint32_t SMEM_KV = 2 * TILE_BYTES;
  static constexpr uint32_t SMEM_STG = SMEM_KV + NS * TILE_BYTES;
  static constexpr uint32_t SMEM_MISC = SMEM_STG + 8 * STG_WARP;  // barriers, TMEM slot, queue
  static constexpr uint32_t MISC_BYTES = 512;
  static constexpr uint32_t MISC_QUEUE = 320;            // QD entries of 8 int32 (32 bytes)
  static constexpr uint32_t SMEM_SEG = SMEM_MISC + MISC_BYTES;  // int32 pairs, then u16 ids
  static constexpr uint32_t SMEM_TOTAL = SMEM_SEG + MAXSEG * 6 + 1024;
  static_assert(SMEM_TOTAL <= 232448, "shared memory per CTA");
  static_assert(MISC_QUEUE + QD * 32 <= MISC_BYTES, "queue region");
  static_assert(!E8 || D == 128, "8-bit inputs: D = 128 (one 128-byte swizzle atom per row)");
  static constexpr int THREADS = 384;
  // Register split (setmaxnreg): launched at 168 per thread (384 x 168 = 64512); warps 8-11
  // give theirs down to REGS_OTHER so that the two softmax warpgroups can take REGS_SOFTMAX.
  // 256 * REGS_SOFTMAX + 128 * REGS_OTHER must not exceed 64512.
  static constexpr int REGS_SOFTMAX = E8 ? 216 : 208;
  static constexpr int REGS_OTHER = E8 ? 72 : 80;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_O = 256;                 // O_h at TM_O + h*D
};

// A decoded work item as handed from the scheduler to the other roles (8 x int32 in the queue).
struct FwdItem {
  int q0, lq, k0, lk, tok0, hb, n_kv0, n_kv1;  // hb < 0: end of this CTA's list
};

__device__ __forceinline__ int lds_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ int lds_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr) : "memory");
  return static_cast<int>(v);
}
__device__ __forceinline__ void sts_s32(uint32_t addr, int v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sts_u16(uint32_t addr, int v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(static_cast<unsigned short>(v))
               : "memory");
}

__device__ __forceinline__ int fwd_group_of(const FwdParams& p, int hb) {
  return static_cast<int>((static_cast<unsigned long long>(hb) * p.g_mul) >> 32);
}

// Number of query-tile pairs of segment s (from cu_seqlens_q in global memory; a negative
// length counts as empty).
__device__ __forceinline__ int fwd_seg_pairs(const FwdParams& p, int s) {
  const int lq = max(__ldg(p.cu_q + s + 1) - __ldg(p.cu_q + s), 0);
  return (lq >> p.log2_tpp) + ((lq & ((1 << p.log2_tpp) - 1)) != 0 ? 1 : 0);
}

// Position of the scheduler in the live-item list. Ranked: `lvl` is the pair index of the
// current level and `cnt` the number of segments live at it (a prefix of the ranking).
// Unranked (more segments than fit in shared memory; segment-major order): `lvl` is the
// current segment and `cnt` its number of pairs. `base` is the list index of the first item of
// the current level or segment, `k` the CTA's next round.
struct FwdWalk {
  long long base;
  int lvl, cnt, k;
};

__device__ __forceinline__ void fwd_walk_init(const FwdParams& p, FwdWalk& w, bool ranked,
                                              uint32_t s_np) {
  w.base = 0;
  w.k = 0;
  if (ranked) {
    w.lvl = lds_s32(s_np) - 1;
    w.cnt = 0;
    while (w.cnt < p.n_seqs && lds_s32(s_np + 4u * w.cnt) > w.lvl) ++w.cnt;
  } else {
    w.lvl = 0;
    w.cnt = fwd_seg_pairs(p, 0);
  }
}

// The CTA's next live item (segment, pair index, head block); false at the end of its list.
__device__ __forceinline__ bool fwd_walk_next(const FwdParams& p, FwdWalk& w, bool ranked,
                                              uint32_t s_np, uint32_t s_id, int& seg, int& pair,
                                              int& hb) {
  const long long G = gridDim.x;
  const long long b = blockIdx.x;
  const long long i = static_cast<long long>(w.k) * G + ((w.k & 1) ? (G - 1 - b) : b);
  ++w.k;
  const long long nhb = p.n_hb;
  if (ranked) {
    while (w.lvl >= 0 && i >= w.base + w.cnt * nhb) {
      w.base += w.cnt * nhb;
      --w.lvl;
      while (w.cnt < p.n_seqs && lds_s32(s_np + 4u * w.cnt) > w.lvl) ++w.cnt;
    }
    if (w.lvl < 0) return false;
    const int o = static_cast<int>(i - w.base);
    const int rank = o / p.n_hb;
    hb = o - rank * p.n_hb;
    seg = lds_u16(s_id + 2u * rank);
    pair = w.lvl;
  } else {
    while (w.lvl < p.n_seqs && i >= w.base + w.cnt * nhb) {
      w.base += w.cnt * nhb;
      ++w.lvl;
      w.cnt = w.lvl < p.n_seqs ? fwd_seg_pairs(p, w.lvl) : 0;
    }
    if (w.lvl >= p.n_seqs) return false;
    const long long o = i - w.base;
    const long long r = o / nhb;
    hb = static_cast<int>(o - r * nhb);
    seg = w.lvl;
    pair = w.cnt - 1 - static_cast<int>(r);
  }
  return true;
}

__device__ __forceinline__ FwdItem fwd_make_item(const FwdParams& p, int seg, int pair, int hb,
                                                 bool causal) {
  FwdItem it;
  it.q0 = __ldg(p.cu_q + seg);
  it.lq = max(__ldg(p.cu_q + seg + 1) - it.q0, 0);
  it.k0 = __ldg(p.cu_k + seg);
  it.lk = max(__ldg(p.cu_k + seg + 1) - it.k0, 0);
  it.tok0 = pair << p.log2_tpp;
  it.hb = hb;
  int n[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int first = it.tok0 + h * p.tok_per_tile;
    int kv_end = 0;
    if (h < p.subtiles && first < it.lq) {
      kv_end = it.lk;
      if (causal) {
        const int last = min(first + p.tok_per_tile, it.lq) - 1;
        kv_end = min(it.lk, last + 1 + it.lk - it.lq);
      }
    }
    n[h] = kv_end > 0 ? (kv_end + 127) / 128 : 0;
  }
  it.n_kv0 = n[0];
  it.n_kv1 = n[1];
  return it;
}

__device__ __forceinline__ FwdItem fwd_read_item(uint32_t e) {
  FwdItem it;
  it.q0 = lds_s32(e);
  it.lq = lds_s32(e + 4);
  it.k0 = lds_s32(e + 8);
  it.lk = lds_s32(e + 12);
  it.tok0 = lds_s32(e + 16);
  it.hb = lds_s32(e + 20);
  it.n_kv0 = lds_s32(e + 24);
  it.n_kv1 = lds_s32(e + 28);
  return it;
}

__device__ __forceinline__ void fwd_write_item(uint32_t e, const FwdItem& it) {
  sts_s32(e, it.q0);
  sts_s32(e + 4, it.lq);
  sts_s32(e + 8, it.k0);
  sts_s32(e + 12, it.lk);
  sts_s32(e + 16, it.tok0);
  sts_s32(e + 20, it.hb);
  sts_s32(e + 24, it.n_kv0);
  sts_s32(e + 28, it.n_kv1);
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

// Maximum of 128 values (four independent 3-input max chains).
__device__ __forceinline__ float row_max128(const float (&x)[128]) {
  float a0 = x[0], a1 = x[1], a2 = x[2], a3 = x[3];
#pragma unroll
  for (int i = 0; i < 15; ++i) {
    a0 = max3f(a0, x[8 + 8 * i + 0], x[8 + 8 * i + 1]);
    a1 = max3f(a1, x[8 + 8 * i + 2], x[8 + 8 * i + 3]);
    a2 = max3f(a2, x[8 + 8 * i + 4], x[8 + 8 * i + 5]);
    a3 = max3f(a3, x[8 + 8 * i + 6], x[8 + 8 * i + 7]);
  }
  a0 = max3f(a0, x[4], x[5]);
  a1 = max3f(a1, x[6], x[7]);
  return fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
}

// Maximum over the row of c1*S(c) (+ slope2*c with ALiBi), without the per-tile constant.
template <bool ALIBI>
__device__ __forceinline__ float tile_score_max(const float (&x)[128], float c1, float slope2) {
  if constexpr (!ALIBI) {
    return row_max128(x) * c1;
  } else {
    const uint64_t c1x2 = f2_pack(c1, c1);
    const uint64_t inc = f2_pack(2.f * slope2, 2.f * slope2);
    float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
    for (int c32 = 0; c32 < 4; ++c32) {
      uint64_t cb = f2_pack(slope2 * static_cast<float>(c32 * 32),
                            slope2 * static_cast<float>(c32 * 32 + 1));
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int c = c32 * 32 + 2 * i;
        float e0, e1;
        f2_unpack(f2_fma(f2_pack(x[c], x[c + 1]), c1x2, cb), e0, e1);
        if (i & 1)
          m1 = max3f(m1, e0, e1);
        else
          m0 = max3f(m0, e0, e1);
        cb = f2_add(cb, inc);
      }
    }
    return fmaxf(m0, m1);
  }
}

// Two values as e4m3 (round to nearest even, saturating), the first in the low byte.
__device__ __forceinline__ uint32_t fp8x2_e4m3(float lo, float hi) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE,
                                                         __NV_E4M3));
}

// p(c) = 2^(c1*x(c) + slope2*c - off) (slope2 term only with ALiBi) for the 128 columns of this
// thread's row, packed to 16-bit pairs over the first 64 TMEM columns at t_s (E8: to e4m3
// quadruples over the first 32 columns). Returns the row sum of p in fp32. (No running maximum
// is kept here: the softmax issue slots are the scarce resource, and the sum alone tells
// whether any p exceeded the caller's bound.)
template <bool BF16, bool ALIBI, bool E8 = false>
__device__ __forceinline__ float exp_tile_to_tmem(const float (&x)[128], float c1, float slope2,
                                                  float off, uint32_t t_s) {
  const uint64_t c1x2 = f2_pack(c1, c1);
  const uint64_t inc = f2_pack(2.f * slope2, 2.f * slope2);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) {
    uint64_t cb = ALIBI ? f2_pack(slope2 * static_cast<float>(c4 * 32) - off,
                                  slope2 * static_cast<float>(c4 * 32 + 1) - off)
                        : f2_pack(-off, -off);
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = c4 * 32 + 2 * i;
      float e0, e1;
      f2_unpack(f2_fma(f2_pack(x[c], x[c + 1]), c1x2, cb), e0, e1);
      if (ALIBI) cb = f2_add(cb, inc);
      const float p0 = ex2_approx(e0);
      const float p1 = ex2_approx(e1);
      acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
      if constexpr (E8) {
        const uint32_t two = fp8x2_e4m3(p0, p1);
        if (i & 1)
          pk[i >> 1] |= two << 16;
        else
          pk[i >> 1] = two;
      } else {
        pk[i] = pack2<BF16>(p0, p1);
      }
    }
    if constexpr (E8)
      tmem_st8(t_s + c4 * 8, *reinterpret_cast<const uint32_t(*)[8]>(&pk[0]));
    else
      tmem_st16(t_s + c4 * 16, pk);
  }
  const uint64_t t = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  float r0, r1;
  f2_unpack(t, r0, r1);
  return r0 + r1;
}

// One key tile of the online softmax for this thread's row (= TMEM lane): loads the 128 scores
// of S from TMEM at t_s, applies scale, ALiBi and the mask, updates the running maximum m_ref and
// sum l, and writes P (16-bit pairs, or e4m3 quadruples) over the first columns of S. Returns
// true when O must be rescaled by alpha before this tile's P V.
//   kv0: key index of column 0; pos: key position of the row; p_min: that of the sub-tile's
//   first row (rows are ordered by token, so it bounds the diagonal of the whole sub-tile).
template <bool BF16, bool CAUSAL, bool ALIBI, bool E8, bool FOLD = (ALIBI && !E8)>
__device__ __forceinline__ bool fwd_softmax_tile(const FwdParams& p, uint32_t t_s, int kv0,
                                                 int lk, int pos, int p_min, float slope2,
                                                 float& m_ref, float& l, float& alpha) {
  uint32_t sr[128];
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4)
    tmem_ld32(t_s + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c4 * 32]));
  tmem_wait_ld();
  const bool need_mask = (kv0 + 128 > lk) || (CAUSAL && kv0 + 127 > p_min);
  const int limit = (CAUSAL ? min(pos, lk - 1) : lk - 1) - kv0;
  float x[128];
#pragma unroll
  for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(sr[c]);
  // Row maximum of this tile (log2 units) and the exponent offset for this tile:
  //   fast path, no ALiBi:      x = S (raw), score = c1*x,        p = 2^(c1*x - m_ref)
  //   fast path, causal ALiBi:  x = c1*S + slope2*c, score = x + K with the row/tile
  //                             constant K = slope2*(kv0 - pos), p = 2^(x - (m_ref - K))
  //   general path:             x = score,                        p = 2^(x - m_ref)
  const bool fast = (p.c1 > 0.f) && (!ALIBI || CAUSAL);
  float kconst = 0.f;
  bool resc = false;
  alpha = 1.f;
  if (fast) {
    // score(c) = c1*S(c) + slope2*c + kconst; exponent e(c) = score(c) - m_ref is formed in
    // one packed FMA per column pair: e = c1*S + (slope2*c - off), off = m_ref - kconst.
    if constexpr (ALIBI) kconst = slope2 * static_cast<float>(kv0 - pos);
    if (need_mask) {
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if (c > limit) x[c] = -INFINITY;
    }
    // Tiles are visited diagonal-first, so once a reference maximum exists the next tile
    // rarely takes p out of range: exponentiate against it straight away and redo the tile in
    // the rare case it does. The first tile of a row takes its maximum first.
    const bool speculate = __all_sync(0xffffffffu, m_ref != -INFINITY);
    // Every p of the tile is at most its row sum, so a sum within the bound keeps every p within
    // the range P is packed into: 2^15 for 16-bit P (f16 holds up to 65504; bf16 has fp32's
    // range), 2^8 for e4m3 (448). Otherwise (rare: key tiles are visited from the diagonal down)
    // take the tile's true maximum and redo the tile against it. The bound only limits how far
    // the reference maximum may lag; O and l stay in fp32 either way. (The first tile's maximum
    // applies the lazy threshold; a redo adopts any larger maximum.)
    float rs;
    if constexpr (FOLD) {
      // Both passes in one loop, so that the exponential step is emitted once; measured faster
      // with ALiBi and 16-bit P at head dim 128 and in the 256-wide kernel, slower for the other
      // 128-wide variants, which keep the two calls below.
      bool take_max = !speculate;
      rs = 0.f;
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        if (take_max) {
          const float m_tile = tile_score_max<ALIBI>(x, p.c1, slope2) + kconst;
          const float m_new = fmaxf(m_ref, m_tile);
          if (pass == 0 ? m_new > m_ref + 8.0f : m_tile > m_ref) {
            resc = true;
            alpha = ex2_approx(m_ref - m_new);
            l *= alpha;
            m_ref = m_new;
          }
        }
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        rs = exp_tile_to_tmem<BF16, ALIBI, E8>(x, p.c1, slope2, m_use - kconst, t_s);
        if (take_max || !__any_sync(0xffffffffu, rs > (E8 ? 256.0f : 32768.0f))) break;
        take_max = true;
      }
    } else {
      if (!speculate) {
        const float m_tile = tile_score_max<ALIBI>(x, p.c1, slope2) + kconst;
        const float m_new = fmaxf(m_ref, m_tile);
        resc = m_new > m_ref + 8.0f;
        if (resc) {
          alpha = ex2_approx(m_ref - m_new);
          l *= alpha;
          m_ref = m_new;
        }
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      rs = exp_tile_to_tmem<BF16, ALIBI, E8>(x, p.c1, slope2, m_use - kconst, t_s);
      if (speculate) {
        const bool over = rs > (E8 ? 256.0f : 32768.0f);
        if (__any_sync(0xffffffffu, over)) {
          const float m_tile = tile_score_max<ALIBI>(x, p.c1, slope2) + kconst;
          if (m_tile > m_ref) {
            resc = true;
            alpha = ex2_approx(m_ref - m_tile);
            l *= alpha;
            m_ref = m_tile;
          }
          rs = exp_tile_to_tmem<BF16, ALIBI, E8>(x, p.c1, slope2, m_ref - kconst, t_s);
        }
      }
    }
    l += rs;
  } else {
    const float dd0 = static_cast<float>(kv0 - pos);
#pragma unroll
    for (int c = 0; c < 128; ++c) {
      float v = x[c] * p.c1;
      if constexpr (ALIBI) v = fmaf(-slope2, fabsf(dd0 + static_cast<float>(c)), v);
      if (need_mask && c > limit) v = -INFINITY;
      x[c] = v;
    }
    const float m_tile = row_max128(x);
    const float m_new = fmaxf(m_ref, m_tile);
    resc = m_new > m_ref + 8.0f;
    if (resc) {
      alpha = ex2_approx(m_ref - m_new);
      l *= alpha;
      m_ref = m_new;
    }
    const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
    l += exp_tile_to_tmem<BF16, false, E8>(x, 1.f, 0.f, m_use, t_s);
  }
  return resc;
}

// End of a role: every thread of the CTA arrives here (from its own code path) before the
// tcgen05 issuer warp releases tensor memory.
__device__ __forceinline__ void fwd_teardown(bool owner, uint32_t tmem, uint32_t ncols) {
  tc_fence_before();
  asm volatile("bar.sync 0;" ::: "memory");
  if (owner) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// BF16 selects the 16-bit type of q/k/v/out (bf16 or f16); with E8, q/k/v are e4m3 and out is
// the BF16-selected 16-bit type. tm_o maps out with a box of one warp's 32 rows x 64 columns.
template <int D, bool BF16, bool CAUSAL, bool ALIBI, bool E8 = false>
__global__ void __launch_bounds__(384, 1)
    mea_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using C = FwdCfg<D, E8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_s = sbase + C::SMEM_Q;
  const uint32_t kv_s0 = sbase + C::SMEM_KV;

  constexpr int B_QF = 0, B_QE = 1, B_KVF = 2, B_KVE = 2 + C::NS, B_SF = 2 + 2 * C::NS;
  constexpr int B_PF = B_SF + 2, B_OF = B_PF + 2, B_OE = B_OF + 2, B_DR = B_OE + 2;
  constexpr int B_IF = B_DR + 1, B_IE = B_IF + C::QD;
  constexpr int N_BARS = B_IE + C::QD;
  static_assert(8 * N_BARS + 8 <= C::MISC_QUEUE, "barrier region");
  const uint32_t bar0 = sbase + C::SMEM_MISC;
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC + 8 * N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t queue = sbase + C::SMEM_MISC + C::MISC_QUEUE;
  const uint32_t s_np = sbase + C::SMEM_SEG;           // int32[MAXSEG]: pairs, by rank
  const uint32_t s_id = s_np + 4u * C::MAXSEG;         // u16[MAXSEG]: segment, by rank

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t tmo = p.timeout_ns;
  const unsigned ecode = KID_FWD << 8;

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_QF), 1);
    mbar_init(BAR(B_QE), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(BAR(B_KVF + s), 1);
      mbar_init(BAR(B_KVE + s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(BAR(B_SF + h), 1);
      mbar_init(BAR(B_PF + h), 4);  // one elected arrival per softmax warp
      mbar_init(BAR(B_OF + h), 1);
      mbar_init(BAR(B_OE + h), 128);
    }
    mbar_init(BAR(B_DR), 1);
    for (int s = 0; s < C::QD; ++s) {
      mbar_init(BAR(B_IF + s), 1);
      mbar_init(BAR(B_IE + s), 9);  // the issuer and one elected lane per softmax warp
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  // Rank the segments by their number of query-tile pairs (descending, ties by index): the
  // scheduler's levels then hold a prefix of the ranking. The staging area holds the unranked
  // counts meanwhile (it is not used before the first epilogue).
  const bool ranked = p.n_seqs <= C::MAXSEG;
  if (ranked) {
    const uint32_t tmp = sbase + C::SMEM_STG;
    for (int s = threadIdx.x; s < p.n_seqs; s += blockDim.x) sts_s32(tmp + 4u * s, fwd_seg_pairs(p, s));
    __syncthreads();
    for (int s = threadIdx.x; s < p.n_seqs; s += blockDim.x) {
      const int key = lds_s32(tmp + 4u * s);
      int rank = 0;
      for (int t = 0; t < p.n_seqs; ++t) {
        const int v = lds_s32(tmp + 4u * t);
        rank += (v > key || (v == key && t < s)) ? 1 : 0;
      }
      sts_s32(s_np + 4u * rank, key);
      sts_u16(s_id + 2u * rank, s);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  static_assert(256 * C::REGS_SOFTMAX + 128 * C::REGS_OTHER <= 384 * 168, "register split");
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_OTHER));
    if (warp == 9) {
    // ---------------------------------------------------------------- scheduler + TMA producer
    if (lane == 0) {
      uint32_t kv_cnt = 0, q_cnt = 0, it_cnt = 0;
      bool ok = true;
      const uint64_t pol_once = l2_policy_evict_first(), pol_reuse = l2_policy_evict_last();
      FwdWalk w;
      fwd_walk_init(p, w, ranked, s_np);
      int seg = 0, pair = 0, hb = 0;
      bool have = fwd_walk_next(p, w, ranked, s_np, s_id, seg, pair, hb);
      FwdItem cur{};
      if (have) cur = fwd_make_item(p, seg, pair, hb, CAUSAL);
      while (ok) {
        // Hand the item (or the end of the list) to the issuer and the softmax warps.
        const uint32_t slot = it_cnt % C::QD;
        ok = mbar_wait(BAR(B_IE + slot), ((it_cnt / C::QD) & 1u) ^ 1u, abort_flag, tmo, ecode | 12);
        if (!ok) break;
        if (!have) cur.hb = -1;
        fwd_write_item(queue + 32u * slot, cur);
        mbar_arrive(BAR(B_IF + slot));
        ++it_cnt;
        if (!have) break;
        FwdItem nxt{};
        const bool have2 = fwd_walk_next(p, w, ranked, s_np, s_id, seg, pair, hb);
        if (have2) nxt = fwd_make_item(p, seg, pair, hb, CAUSAL);
        const int nmax = max(cur.n_kv0, cur.n_kv1);
        if (nmax > 0) {
          const int g = fwd_group_of(p, cur.hb);
          ok = mbar_wait(BAR(B_QE), (q_cnt & 1u) ^ 1u, abort_flag, tmo, ecode | 1);
          if (!ok) break;
          mbar_arrive_expect_tx(BAR(B_QF), 2 * C::TILE_BYTES);
          // Q is read by this item alone: evict-first, so that the K/V tiles that the other
          // items of the segment read again stay in L2 (evict-last below).
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int a = 0; a < C::ATOMS; ++a)
              tma_load_3d_hint(q_s + h * C::TILE_BYTES + a * C::ATOM_BYTES, &tm_q, BAR(B_QF),
                               a * C::ATOM_COLS, cur.hb << p.log2_p,
                               cur.q0 + cur.tok0 + h * p.tok_per_tile, pol_once);
          ++q_cnt;
          for (int j = 0; j < nmax && ok; ++j) {
#pragma unroll 1
            for (int kv = 0; kv < 2; ++kv) {
              const uint32_t s = kv_cnt % C::NS;
              const uint32_t ph = (kv_cnt / C::NS) & 1u;
              ok = mbar_wait(BAR(B_KVE + s), ph ^ 1u, abort_flag, tmo, ecode | 2);
              if (!ok) break;
              mbar_arrive_expect_tx(BAR(B_KVF + s), C::TILE_BYTES);
              const uint32_t dst = kv_s0 + s * C::TILE_BYTES;
#pragma unroll
              for (int a = 0; a < C::ATOMS; ++a)
                tma_load_3d_hint(dst + a * C::ATOM_BYTES, kv ? &tm_v : &tm_k, BAR(B_KVF + s),
                                 a * C::ATOM_COLS, g, cur.k0 + (nmax - 1 - j) * 128, pol_reuse);
              ++kv_cnt;
            }
          }
          // Warm L2 with the next item's Q tiles and its first two K/V tiles while this item's
          // last steps are still being computed: the next Q can only be loaded once this
          // item's last Q K^T has finished, and fetched cold from HBM it would stall the item
          // boundary.
          const int nm = max(nxt.n_kv0, nxt.n_kv1);
          if (ok && have2 && nm > 0) {
            const int ng = fwd_group_of(p, nxt.hb);
#pragma unroll
            for (int a = 0; a < C::ATOMS; ++a) {
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_prefetch_l2_3d(&tm_q, a * C::ATOM_COLS, nxt.hb << p.log2_p,
                                   nxt.q0 + nxt.tok0 + h * p.tok_per_tile);
              for (int j = 0; j < min(nm, 2); ++j) {
                tma_prefetch_l2_3d(&tm_k, a * C::ATOM_COLS, ng, nxt.k0 + (nm - 1 - j) * 128);
                tma_prefetch_l2_3d(&tm_v, a * C::ATOM_COLS, ng, nxt.k0 + (nm - 1 - j) * 128);
              }
            }
          }
        }
        cur = nxt;
        have = have2;
      }
      if (!ok) {
        // Let the loads already issued land before the CTA's shared memory goes away.
        for (uint32_t s = 0; s < C::NS && s < kv_cnt; ++s) {
          const uint32_t last = kv_cnt - 1 - ((kv_cnt - 1 - s) % C::NS);
          volatile int never = 0;
          mbar_wait(BAR(B_KVF + s), (last / C::NS) & 1u, &never, tmo, ecode | 15);
        }
        if (q_cnt > 0) {
          volatile int never = 0;
          mbar_wait(BAR(B_QF), (q_cnt - 1) & 1u, &never, tmo, ecode | 15);
        }
      }
    }
    } else if (warp == 8) {
    // ---------------------------------------------------------------- tcgen05 issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = E8 ? umma_idesc_e4m3(128, 128, false, false)
                                       : umma_idesc_f16(BF16, 128, 128, false, false);
      constexpr uint32_t IDESC_PV = E8 ? umma_idesc_e4m3(128, D, false, true)
                                       : umma_idesc_f16(BF16, 128, D, false, true);
      uint32_t kv_cnt = 0, q_cnt = 0, it_cnt = 0;
      uint32_t pv_cnt[2] = {0, 0}, oe_cnt[2] = {0, 0};
      bool ok = true;
      while (ok) {
        const uint32_t slot = it_cnt % C::QD;
        ok = mbar_wait(BAR(B_IF + slot), (it_cnt / C::QD) & 1u, abort_flag, tmo, ecode | 13);
        if (!ok) break;
        const FwdItem it = fwd_read_item(queue + 32u * slot);
        mbar_arrive(BAR(B_IE + slot));
        ++it_cnt;
        if (it.hb < 0) break;
        const int n_kv[2] = {it.n_kv0, it.n_kv1};
        const int nmax = max(n_kv[0], n_kv[1]);
        if (nmax == 0) continue;
        ok = mbar_wait(BAR(B_QF), q_cnt & 1u, abort_flag, tmo, ecode | 6);
        if (!ok) break;
        tc_fence_after();
        const uint32_t base = kv_cnt;
        for (int j = 0; j <= nmax && ok; ++j) {
          const uint32_t ks = (base + 2 * j) % C::NS;
          const uint32_t vs = (base + 2 * j - 1) % C::NS;  // slot of V_{j-1} (j >= 1)
          if (j < nmax) {
            ok = mbar_wait(BAR(B_KVF + ks), ((base + 2 * j) / C::NS) & 1u, abort_flag, tmo,
                           ecode | 7);
            if (!ok) break;
            tc_fence_after();
          }
          bool v_ready = false;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // Tiles are visited from the last (diagonal) one down to tile 0, so the largest
            // scores come first and the lazy O rescale rarely fires. Sub-tile h joins at
            // iteration first_h = nmax - n_h (its own last tile).
            const int first_h = nmax - n_kv[h];
            if (j >= first_h + 1 && n_kv[h] > 0) {
              // ---- O_h += P_h(j-1) V_{j-1}
              if (!v_ready) {
                ok = mbar_wait(BAR(B_KVF + vs), ((base + 2 * j - 1) / C::NS) & 1u, abort_flag,
                               tmo, ecode | 5);
                if (!ok) break;
                v_ready = true;
              }
              ok = mbar_wait_spin(BAR(B_PF + h), pv_cnt[h] & 1u, abort_flag, tmo, ecode | 3);
              if (!ok) break;
              if (j == first_h + 1) {
                ok = mbar_wait(BAR(B_OE + h), (oe_cnt[h] & 1u) ^ 1u, abort_flag, tmo, ecode | 4);
                if (!ok) break;
                ++oe_cnt[h];
              }
              tc_fence_after();
              const uint32_t vbase = kv_s0 + vs * C::TILE_BYTES;
#pragma unroll
              for (int kk = 0; kk < C::BN / C::KSTEP; ++kk) {
                // V rows kk*KSTEP.. (128-byte rows), P columns kk*8.. (32 bytes per row)
                const uint64_t bd =
                    umma_desc_sw128(vbase + kk * C::KSTEP * 128, C::ATOM_BYTES, 1024);
                mma_ts_k<E8>(tmem + C::TM_O + h * D, tmem + h * 128 + kk * 8, bd, IDESC_PV,
                             (j == first_h + 1 && kk == 0) ? 0u : 1u);
              }
              ++pv_cnt[h];
              if (j == nmax) mma_commit(BAR(B_OF + h));
            }
            if (j < nmax && j >= first_h && n_kv[h] > 0) {
              // ---- S_h = Q_h K_j^T
              const uint32_t kbase = kv_s0 + ks * C::TILE_BYTES;
              const uint32_t qbase = q_s + h * C::TILE_BYTES;
#pragma unroll
              for (int kk = 0; kk < D / C::KSTEP; ++kk) {
                const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
                const uint64_t ad = umma_desc_sw128(qbase + off, 16, 1024);
                const uint64_t bd = umma_desc_sw128(kbase + off, 16, 1024);
                mma_ss_k<E8>(tmem + h * 128, ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
              }
              mma_commit(BAR(B_SF + h));
            }
          }
          if (!ok) break;
          if (j < nmax) mma_commit(BAR(B_KVE + ks));
          if (j >= 1) mma_commit(BAR(B_KVE + vs));
          if (j == nmax - 1) mma_commit(BAR(B_QE));
        }
        if (!ok) break;
        kv_cnt = base + 2 * nmax;
        ++q_cnt;
      }
      // Every MMA issued so far must finish before TMEM is released.
      mma_commit(BAR(B_DR));
      volatile int never = 0;
      mbar_wait(BAR(B_DR), 0, &never, tmo, ecode | 14);
    }
    }
    fwd_teardown(warp == 8, tmem, C::TMEM_COLS);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
    // ---------------------------------------------------------------- softmax warpgroups
    const int h = warp >> 2;           // sub-tile of this warpgroup
    const int wq = warp & 3;           // TMEM lane quarter of this warp
    const int r = threadIdx.x & 127;   // row within the sub-tile = TMEM lane
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t t_s = t_lane + h * 128;
    const uint32_t t_o = t_lane + C::TM_O + h * D;
    const uint32_t stg = sbase + C::SMEM_STG + static_cast<uint32_t>(warp) * C::STG_WARP;
    const uint64_t pol_once = l2_policy_evict_first();  // out is written once
    constexpr float LOG2E = 1.4426950408889634f;
    constexpr float LN2 = 0.6931471805599453f;
    uint32_t tile = 0, ocnt = 0, it_cnt = 0;
    bool ok = true;
    const bool out_al32 = (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0 && (p.dh & 15) == 0;
    using OutT = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    while (ok) {
      const uint32_t slot = it_cnt % C::QD;
      ok = mbar_wait(BAR(B_IF + slot), (it_cnt / C::QD) & 1u, abort_flag, tmo, ecode | 11);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const FwdItem it = fwd_read_item(queue + 32u * slot);
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_IE + slot));
      ++it_cnt;
      if (it.hb < 0) break;
      const int sub0 = it.tok0 + h * p.tok_per_tile;  // first token of this sub-tile
      const int tok = sub0 + (r >> p.log2_p);
      const int head = (it.hb << p.log2_p) + (r & (p.P - 1));
      const bool row_valid = tok < it.lq;
      const int nh = h ? it.n_kv1 : it.n_kv0;
      OutT* orow = reinterpret_cast<OutT*>(p.out) +
                   (static_cast<size_t>(it.q0 + tok) * p.hq + head) * p.dh;
      if (nh == 0) {
        if (row_valid) {
          uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int i = 0; i < D / 8; ++i)
            if (i < (p.dh >> 3)) reinterpret_cast<uint4*>(orow)[i] = z;
          if (p.lse) p.lse[static_cast<size_t>(head) * p.total_q + it.q0 + tok] = -INFINITY;
        }
        continue;
      }
      const int pos = tok + it.lk - it.lq;      // key position of this query row
      const int p_min = sub0 + it.lk - it.lq;   // position of the sub-tile's first row
      float slope2 = 0.f;
      if constexpr (ALIBI) slope2 = __ldg(p.slopes + head) * LOG2E;
      float m_ref = -INFINITY, l = 0.f;
      for (int jj = 0; jj < nh; ++jj) {
        const int j = nh - 1 - jj;  // key tile, visited from the diagonal downwards
        ok = mbar_wait(BAR(B_SF + h), tile & 1u, abort_flag, tmo, ecode | 8);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float alpha = 1.f;
        const bool resc = fwd_softmax_tile<BF16, CAUSAL, ALIBI, E8>(
            p, t_s, j * 128, it.lk, pos, p_min, slope2, m_ref, l, alpha);
        // O_h holds the tiles visited before this one and its last PV has completed (it was
        // issued before this QK).
        if (jj > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t o[32];
            tmem_ld32(t_o + c4 * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(t_o + c4 * 32, o);
          }
        }
        // Each thread's P stores complete, then one lane per warp publishes the warp's rows.
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_PF + h));
        ++tile;
      }
      if (!ok) break;
      // ---- epilogue: O / l -> out, lse
      ok = mbar_wait(BAR(B_OF + h), ocnt & 1u, abort_flag, tmo, ecode | 10);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++ocnt;
      tc_fence_after();
      const float inv_l = l > 0.f ? p.o_scale / l : 0.f;
      // The whole O row in one round of loads; once they have landed O_h is free for the next
      // item's P V, before any of the stores.
      uint32_t o[D];
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4)
        tmem_ld32(t_o + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&o[c4 * 32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(BAR(B_OE + h));
#pragma unroll
      for (int i = 0; i < D / 2; ++i)
        o[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
      if (row_valid && p.lse)
        p.lse[static_cast<size_t>(head) * p.total_q + it.q0 + tok] =
            l > 0.f ? (m_ref + __log2f(l)) * LN2 : -INFINITY;
      // The warp's 32 rows are whole when its last row is inside the segment (rows are ordered
      // by token): then they go out as TMA stores of [32 rows x 64 columns] boxes, staged in
      // shared memory with the 128-byte swizzle (16-byte chunk c of row i at c ^ (i & 7)).
      const int last_tok = sub0 + ((32 * wq + 31) >> p.log2_p);
      if (last_tok < it.lq) {
        const int c_head = (it.hb << p.log2_p) + ((32 * wq) & (p.P - 1));
        const int c_tok = it.q0 + sub0 + ((32 * wq) >> p.log2_p);
#pragma unroll
        for (int a = 0; a < C::OUT_ATOMS; ++a) {
          if (a * 64 >= p.dh) break;  // no box starts past the row (e4m3 inputs, dh <= 64)
          // The previous box of this warp has been read out of the staging area.
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(stg + lane * 128u + (static_cast<uint32_t>(c ^ (lane & 7)) << 4),
                         o[a * 32 + 4 * c], o[a * 32 + 4 * c + 1], o[a * 32 + 4 * c + 2],
                         o[a * 32 + 4 * c + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d_hint(&tm_o, stg, a * 64, c_head, c_tok, pol_once);
            bulk_commit();
          }
        }
      } else if (row_valid) {
        // Each thread writes its own row (the first dh columns): 32-byte stores fill whole
        // sectors when the rows stay 32-byte aligned (out is, and dh is a multiple of 16).
        if (out_al32) {
#pragma unroll
          for (int i = 0; i < D / 16; ++i)
            if (i < (p.dh >> 4)) st_global_v8(orow + i * 16, &o[8 * i]);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
          for (int i = 0; i < D / 8; ++i)
            if (i < (p.dh >> 3))
              dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
      }
    }
    // The TMA stores issued by this warp have completed before the CTA exits.
    if (lane == 0) bulk_wait_all();
    __syncwarp();
    fwd_teardown(false, tmem, C::TMEM_COLS);
  }
#undef BAR
}

}  // namespace mea
