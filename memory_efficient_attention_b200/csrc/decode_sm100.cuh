// decode_sm100.cuh — split-KV single-token decode and its log-sum-exp merge, for sm_100a.
//
// The split-K attention of "大模型推理加速终极指南" (section 1): each request's keys are cut into
// fixed-size chunks; every (chunk, head block) work item produces a chunk-normalised partial
// output and its log-sum-exp; a second kernel merges the partials of a request by their lse.
//
// Split kernel (persistent, 160 threads, one CTA per SM):
//   warp 4      TMA producer: K and V tiles of 64 keys x D for the item's KV head, NS-slot ring,
//               streamed continuously across work items.
//   warps 0-3   consumers: warp w takes keys [16w, 16w+16) of every tile. S = q K^T and
//               O += P V on mma.sync m16n8k16 (the query rows are the RB <= 16 heads of one KV
//               group, one token each), online softmax in registers; at the end of an item the
//               four warps merge their (m, l, O) through shared memory and write the partial.
// Decode is bound by streaming K/V from HBM (about 8 flop per byte); the small products only need
// to keep up with that stream, which mma.sync does without loading the FMA pipes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace mea {

struct DecParams {
  const void* q;      // [n_seqs, hq, D]
  void* out;          // [n_seqs, hq, D]
  float* lse;         // [hq, n_seqs] or null
  const int32_t* cu_k;         // prefix sums of the requests' key counts
  const float* slopes;
  const int32_t* block_table;  // paged K/V only: [n_seqs, max_blocks] cache block ids
  int block_size;              // paged: keys per cache block (16, 32 or a multiple of 64)
  int max_blocks;              // paged: row length of block_table
  int num_blocks;              // paged: blocks in the cache (ids outside [0, num_blocks) read 0)
  int box5;                    // paged: 1 = one 5-D box per block covers every 64-column atom
                               // (head_dim a multiple of 64), 0 = one 4-D box per atom
  int lay_log2;                // log2 of the rows per shared-memory layout group (see below)
  float* ws_o;        // [n_slots, hq, D]
  float* ws_lse;      // [n_slots, hq]
  int n_seqs;
  int hq;
  int dh;             // head dim of q, k, v and out rows (<= D; the TMA zero-fills the rest)
  int R;              // query heads per KV head
  int RB;             // query heads per work item (<= 16, divides R)
  int n_hb;           // hq / RB
  int chunk;          // keys per chunk, a multiple of 64
  int n_slots;        // upper bound on the number of chunks
  long long n_items;  // n_slots * n_hb
  float c1;           // scale * log2(e)
  unsigned long long timeout_ns;
};

// Shared-memory layout of a K (or V) stage: groups of 2^lay_log2 key rows, each group
// [atom][rows][128 B] with the 128-byte swizzle. Packed K/V and 4-D paged boxes use one group of
// 64 rows ([atom][64 keys]); 5-D paged boxes land one cache block (min(block_size, 64) rows,
// every atom) per group. Address of 16-byte chunk ch (along D) of key row kr:
template <int D>
__device__ __forceinline__ uint32_t dec_row_addr(uint32_t base, int kr, int ch, int lay_log2) {
  const uint32_t lr = 1u << lay_log2;
  return base + static_cast<uint32_t>(kr >> lay_log2) * (lr * (D / 64) * 128u) +
         static_cast<uint32_t>(ch >> 3) * (lr * 128u) + static_cast<uint32_t>(kr & (lr - 1)) * 128u +
         (static_cast<uint32_t>((ch & 7) ^ (kr & 7)) << 4);
}

template <int D, bool PAGED = false>
struct DecCfg {
  static constexpr int BK = 64;                       // keys per tile
  static constexpr int ATOMS = D / 64;
  static constexpr uint32_t ATOM_BYTES = BK * 128;    // 64 keys x 128 B
  static constexpr uint32_t KT_BYTES = BK * D * 2;    // one K (or V) tile
  static constexpr uint32_t STAGE_BYTES = 2 * KT_BYTES;
  // Ring stages: at D = 128 the paged cache takes a sixth (its stages arrive as several smaller
  // boxes, so more of them in flight pay: +2 % on 16-slot blocks), the packed one stays at five
  // (a sixth measured 0.8 % slower there).
  static constexpr int NS = (D == 256) ? 3 : (D == 128) ? (PAGED ? 6 : 5) : 8;
  // The four warps' partial O rows are merged through shared memory MC columns at a time.
  static constexpr int MC = D < 128 ? D : 128;
  static constexpr uint32_t SMEM_RING = 0;
  static constexpr uint32_t SMEM_MERGE = NS * STAGE_BYTES;            // 4 warps x 16 rows x MC
  static constexpr uint32_t MERGE_O_BYTES = 4 * 16 * MC * 4;
  static constexpr uint32_t SMEM_ML = SMEM_MERGE + MERGE_O_BYTES;     // 4 warps x 16 x (m, l)
  static constexpr uint32_t SMEM_BAR = SMEM_ML + 4 * 16 * 2 * 4;
  static constexpr uint32_t SMEM_TOTAL = SMEM_BAR + 256 + 1024;
  static_assert(SMEM_TOTAL <= 232448, "shared memory per CTA");
  static constexpr int THREADS = 160;
};

// Number of chunks of request i.
__device__ __forceinline__ int dec_nchunks(const int32_t* cu, int i, int chunk) {
  const int L = __ldg(cu + i + 1) - __ldg(cu + i);
  return (L + chunk - 1) / chunk;
}

// Warp-cooperative: maps a flat chunk id to (request b, chunk c of b); b = -1 past the end.
__device__ __forceinline__ void dec_find_chunk(const int32_t* cu, int n, int chunk, int cid,
                                               int& b, int& c) {
  const int lane = threadIdx.x & 31;
  int base = 0;
  for (int i0 = 0; i0 < n; i0 += 32) {
    const int i = i0 + lane;
    const int cnt = i < n ? dec_nchunks(cu, i, chunk) : 0;
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    const int excl = incl - cnt;
    const bool hit = (i < n) && cid >= base + excl && cid < base + incl;
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (m) {
      const int src = __ffs(m) - 1;
      b = i0 + src;
      c = cid - base - __shfl_sync(0xffffffffu, excl, src);
      return;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  b = -1;
  c = 0;
}

// Warp-cooperative: first flat chunk id of request b.
__device__ __forceinline__ int dec_chunk_start(const int32_t* cu, int b, int chunk) {
  const int lane = threadIdx.x & 31;
  int acc = 0;
  for (int i0 = 0; i0 < b; i0 += 32) {
    const int i = i0 + lane;
    acc += (i < b) ? dec_nchunks(cu, i, chunk) : 0;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  return acc;
}

// PAGED: K/V live in a block cache [num_blocks, block_size, Hkv, D] addressed through a per-request
// block table (4-D TMA maps) instead of a packed [T_k, Hkv, D] tensor (3-D maps).
template <int D, bool BF16, bool ALIBI, bool PAGED = false>
__global__ void __launch_bounds__(160, 1)
    mea_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const DecParams p) {
  using C = DecCfg<D, PAGED>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = smem_u32(smem);
  float* merge_o = reinterpret_cast<float*>(smem + C::SMEM_MERGE);
  float* merge_ml = reinterpret_cast<float*>(smem + C::SMEM_ML);
  const uint32_t bar0 = sbase + C::SMEM_BAR;
#define DBAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
  // B_M0 / B_M1: the four consumer warps' rendezvous before / after the partial merge.
  constexpr int B_F = 0, B_E = C::NS, B_M0 = 2 * C::NS, B_M1 = B_M0 + 1, N_BARS = B_M1 + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_BAR + 8 * N_BARS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t tmo = p.timeout_ns;
  const unsigned ecode = KID_DECODE << 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(DBAR(B_F + s), 1);
      mbar_init(DBAR(B_E + s), 4);
    }
    mbar_init(DBAR(B_M0), 128);
    mbar_init(DBAR(B_M1), 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    uint32_t cnt = 0;
    bool ok = true;
    for (long long lin = blockIdx.x; lin < p.n_items && ok; lin += gridDim.x) {
      const int cid = static_cast<int>(lin / p.n_hb);
      const int hb = static_cast<int>(lin - static_cast<long long>(cid) * p.n_hb);
      int b, c;
      dec_find_chunk(p.cu_k, p.n_seqs, p.chunk, cid, b, c);
      if (b < 0) break;  // flat chunk ids only grow along this CTA's sequence
      const int k0 = __ldg(p.cu_k + b);
      const int L = __ldg(p.cu_k + b + 1) - k0;
      const int key0 = c * p.chunk;
      const int nk = min(p.chunk, L - key0);
      const int n_tiles = (nk + C::BK - 1) / C::BK;
      const int g = (hb * p.RB) / p.R;
      if constexpr (PAGED) {
        // Tile keys [kt, kt + 64) of request b come from `per` cache blocks: one box per block
        // and per (K or V, 64-column atom) for block sizes 16 and 32 (boxes of block_size rows
        // at row offsets that keep the 128-B swizzle aligned), or a 64-row slice of one block
        // for block sizes that are multiples of 64. The boxes of a stage are issued by as many
        // lanes, each of which also reads its block ids ahead (at 16-slot blocks a
        // stage is 16 boxes of 2 KB, and one lane issuing them all starved the stream). Blocks
        // past the request's last one use id num_blocks, which the TMA fills with zeros.
        const int32_t* row = p.block_table + static_cast<size_t>(b) * p.max_blocks;
        const int bs = p.block_size;
        const int per = bs >= C::BK ? 1 : C::BK / bs;
        const int nblk = min((L + bs - 1) / bs, p.max_blocks);
        // 4-D: one box per (block, K or V, atom), <= 16 per stage; 5-D: one per (block, K or V)
        const int apb = p.box5 ? 1 : C::ATOMS;             // boxes per block and tensor
        const int nbox = per * 2 * apb;
        const int my_i = lane / (2 * apb);                 // block of the tile
        const int my_v = (lane / apb) & 1;                 // K or V
        const int my_a = lane % apb;                       // 64-column atom (4-D)
        const bool issuer = lane < nbox;
        auto block_id = [&](int t) {
          const int j = (key0 + t * C::BK + my_i * bs) / bs;
          return (issuer && t < n_tiles && j < nblk) ? __ldg(row + j) : p.num_blocks;
        };
        // Block ids of tiles t .. t+3: each read is in flight for three tiles before its TMA
        // needs it (a block-table line that misses in L2 waits on HBM under a full load).
        int id_q[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) id_q[u] = block_id(u);
        for (int t = 0; t < n_tiles; ++t) {
          const int id = id_q[0];
          id_q[0] = id_q[1];
          id_q[1] = id_q[2];
          id_q[2] = id_q[3];
          id_q[3] = block_id(t + 4);
          const uint32_t s = cnt % C::NS;
          const uint32_t ph = (cnt / C::NS) & 1u;
          if (lane == 0) {
            ok = mbar_wait(DBAR(B_E + s), ph ^ 1u, abort_flag, tmo, ecode | 1);
            if (ok) mbar_arrive_expect_tx(DBAR(B_F + s), C::STAGE_BYTES);
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          if (issuer) {
            const int r0 = bs >= C::BK ? (key0 + t * C::BK) % bs : 0;
            const uint32_t stg = sbase + C::SMEM_RING + s * C::STAGE_BYTES + my_v * C::KT_BYTES;
            if (p.box5) {
              // the block's rows for every atom: [atom][rows][128 B], one layout group
              const uint32_t dst = stg + static_cast<uint32_t>(my_i * bs * C::ATOMS * 128);
              tma_load_5d(dst, my_v ? &tm_v : &tm_k, DBAR(B_F + s), 0, r0, 0, g, id);
            } else {
              const uint32_t dst = stg + my_a * C::ATOM_BYTES + static_cast<uint32_t>(my_i * bs * 128);
              tma_load_4d(dst, my_v ? &tm_v : &tm_k, DBAR(B_F + s), my_a * 64, g, r0, id);
            }
          }
          ++cnt;
        }
      } else if (lane == 0) {
        for (int t = 0; t < n_tiles; ++t) {
          const uint32_t s = cnt % C::NS;
          const uint32_t ph = (cnt / C::NS) & 1u;
          ok = mbar_wait(DBAR(B_E + s), ph ^ 1u, abort_flag, tmo, ecode | 1);
          if (!ok) break;
          mbar_arrive_expect_tx(DBAR(B_F + s), C::STAGE_BYTES);
          const uint32_t dst = sbase + C::SMEM_RING + s * C::STAGE_BYTES;
          const int tok = k0 + key0 + t * C::BK;
#pragma unroll
          for (int a = 0; a < C::ATOMS; ++a) {
            tma_load_3d(dst + a * C::ATOM_BYTES, &tm_k, DBAR(B_F + s), a * 64, g, tok);
            tma_load_3d(dst + C::KT_BYTES + a * C::ATOM_BYTES, &tm_v, DBAR(B_F + s), a * 64,
                        g, tok);
          }
          ++cnt;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      cnt = __shfl_sync(0xffffffffu, cnt, 0);
    }
    if (!ok && lane == 0) {
      for (uint32_t s = 0; s < C::NS && s < cnt; ++s) {
        const uint32_t last = cnt - 1 - ((cnt - 1 - s) % C::NS);
        volatile int never = 0;
        mbar_wait(DBAR(B_F + s), (last / C::NS) & 1u, &never, tmo, ecode | 15);
      }
    }
  } else {
    // ------------------------------------------------------------------ consumers (warps 0-3)
    constexpr float LOG2E = 1.4426950408889634f;
    constexpr float LN2 = 0.6931471805599453f;
    const int g8 = lane >> 2;  // fragment row (head) 0..7
    const int t4 = lane & 3;   // fragment column pair
    uint32_t cnt = 0, n_done = 0, m_cnt = 0;
    bool ok = true;
    for (long long lin = blockIdx.x; lin < p.n_items && ok; lin += gridDim.x) {
      const int cid = static_cast<int>(lin / p.n_hb);
      const int hb = static_cast<int>(lin - static_cast<long long>(cid) * p.n_hb);
      int b, c;
      dec_find_chunk(p.cu_k, p.n_seqs, p.chunk, cid, b, c);
      if (b < 0) break;
      const int L = __ldg(p.cu_k + b + 1) - __ldg(p.cu_k + b);
      const int key0 = c * p.chunk;
      const int nk = min(p.chunk, L - key0);
      const int n_tiles = (nk + C::BK - 1) / C::BK;
      const int pos = L - 1;  // the query is the newest token of its request
      // q fragments: rows g8 and g8+8 are heads hb*RB + row (zero when row >= RB).
      const int h_lo = hb * p.RB + g8, h_hi = hb * p.RB + g8 + 8;
      const bool v_lo = g8 < p.RB, v_hi = g8 + 8 < p.RB;
      // Columns past dh are zero (as are the K/V columns the TMA fills past dh).
      uint32_t qa[D / 16][4];
      {
        const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q);
        const int dw = p.dh >> 1;  // 32-bit words per row
        const size_t rlo = (static_cast<size_t>(b) * p.hq + h_lo) * dw;
        const size_t rhi = (static_cast<size_t>(b) * p.hq + h_hi) * dw;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const bool c0 = kk * 8 + t4 < dw, c1 = kk * 8 + 4 + t4 < dw;
          qa[kk][0] = (v_lo && c0) ? __ldg(q32 + rlo + kk * 8 + t4) : 0u;
          qa[kk][1] = (v_hi && c0) ? __ldg(q32 + rhi + kk * 8 + t4) : 0u;
          qa[kk][2] = (v_lo && c1) ? __ldg(q32 + rlo + kk * 8 + 4 + t4) : 0u;
          qa[kk][3] = (v_hi && c1) ? __ldg(q32 + rhi + kk * 8 + 4 + t4) : 0u;
        }
      }
      float sl_lo = 0.f, sl_hi = 0.f;
      if constexpr (ALIBI) {
        sl_lo = v_lo ? __ldg(p.slopes + h_lo) * LOG2E : 0.f;
        sl_hi = v_hi ? __ldg(p.slopes + h_hi) * LOG2E : 0.f;
      }
      float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
      float o[D / 8][4];
#pragma unroll
      for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

      for (int t = 0; t < n_tiles; ++t) {
        const uint32_t s = cnt % C::NS;
        const uint32_t ph = (cnt / C::NS) & 1u;
        ok = mbar_wait(DBAR(B_F + s), ph, abort_flag, tmo, ecode | 2);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const uint32_t kst = sbase + C::SMEM_RING + s * C::STAGE_BYTES;
        const uint32_t vst = kst + C::KT_BYTES;
        bool zeroed = false;
        if constexpr (PAGED) {
          // A cache block's slots past the sequence end may hold anything (0 * NaN is NaN in
          // P V): zero this warp's V rows past the last key of a partial tile.
          const int valid = nk - t * C::BK;
          if (valid < C::BK) {
            const int r_lo = max(valid, warp * 16), r_hi = warp * 16 + 16;
            for (int i = lane; i < (r_hi > r_lo ? (r_hi - r_lo) * (D / 8) : 0); i += 32) {
              const int rr = r_lo + i / (D / 8), ch = i % (D / 8);
              const uint32_t addr = dec_row_addr<D>(vst, rr, ch ^ (rr & 7), p.lay_log2);
              asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u)
                           : "memory");
            }
            zeroed = true;
            __syncwarp();
          }
        }
        // ---- S^T fragment: rows = heads, cols = this warp's 16 keys (two n-tiles of 8)
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
          const int kr = warp * 16 + ((lane >> 4) << 3) + (lane & 7);  // key row in the tile
          const int csel = (lane >> 3) & 1;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int ch = 2 * kk + csel;  // 16-byte chunk along D
            const uint32_t addr = PAGED ? dec_row_addr<D>(kst, kr, ch, p.lay_log2)
                                        : kst + (ch >> 3) * C::ATOM_BYTES + kr * 128 +
                                              ((((ch & 7) ^ (kr & 7))) << 4);
            uint32_t r0, r1, r2, r3;
            ldsm_x4(addr, r0, r1, r2, r3);
            mma16816<BF16>(sc[0], qa[kk], r0, r1);
            mma16816<BF16>(sc[1], qa[kk], r2, r3);
          }
        }
        // ---- online softmax over the 16 keys (rows g8 / g8+8)
        const int kbase = key0 + t * C::BK + warp * 16;  // key index (in request) of col 0
        float x[2][4];
        float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
        for (int n = 0; n < 2; ++n) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = kbase + n * 8 + 2 * t4 + e;
            const bool kv = key < key0 + nk;
            float a = sc[n][e] * p.c1, bb = sc[n][2 + e] * p.c1;
            if constexpr (ALIBI) {
              const float dist = static_cast<float>(pos - key);
              a = fmaf(-sl_lo, dist, a);
              bb = fmaf(-sl_hi, dist, bb);
            }
            x[n][e] = kv ? a : -INFINITY;
            x[n][2 + e] = kv ? bb : -INFINITY;
            mx_lo = fmaxf(mx_lo, x[n][e]);
            mx_hi = fmaxf(mx_hi, x[n][2 + e]);
          }
        }
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
          mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, off));
          mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, off));
        }
        const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
        const float al_lo = (mn_lo == -INFINITY) ? 1.f : ex2_approx(m_lo - mn_lo);
        const float al_hi = (mn_hi == -INFINITY) ? 1.f : ex2_approx(m_hi - mn_hi);
        const float mu_lo = (mn_lo == -INFINITY) ? 0.f : mn_lo;
        const float mu_hi = (mn_hi == -INFINITY) ? 0.f : mn_hi;
        m_lo = mn_lo;
        m_hi = mn_hi;
        float pr[2][4];
        float s_lo = 0.f, s_hi = 0.f;
#pragma unroll
        for (int n = 0; n < 2; ++n) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            pr[n][e] = ex2_approx(x[n][e] - mu_lo);
            pr[n][2 + e] = ex2_approx(x[n][2 + e] - mu_hi);
            s_lo += pr[n][e];
            s_hi += pr[n][2 + e];
          }
        }
        l_lo = l_lo * al_lo + s_lo;
        l_hi = l_hi * al_hi + s_hi;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          o[n][0] *= al_lo;
          o[n][1] *= al_lo;
          o[n][2] *= al_hi;
          o[n][3] *= al_hi;
        }
        uint32_t pa[4];
        pa[0] = dpack2<BF16>(pr[0][0], pr[0][1]);
        pa[1] = dpack2<BF16>(pr[0][2], pr[0][3]);
        pa[2] = dpack2<BF16>(pr[1][0], pr[1][1]);
        pa[3] = dpack2<BF16>(pr[1][2], pr[1][3]);
        // ---- O += P V over this warp's 16 keys
        {
          const int kr = warp * 16 + (((lane >> 3) & 1) << 3) + (lane & 7);
          const int csel = lane >> 4;
#pragma unroll
          for (int n = 0; n < D / 8; n += 2) {
            const int ch = n + csel;
            const uint32_t addr = PAGED ? dec_row_addr<D>(vst, kr, ch, p.lay_log2)
                                        : vst + (ch >> 3) * C::ATOM_BYTES + kr * 128 +
                                              ((((ch & 7) ^ (kr & 7))) << 4);
            uint32_t r0, r1, r2, r3;
            ldsm_x4_t(addr, r0, r1, r2, r3);
            mma16816<BF16>(o[n], pa, r0, r1);
            mma16816<BF16>(o[n + 1], pa, r2, r3);
          }
        }
        // Generic-proxy writes to the slot must be ordered before the next TMA write into it.
        if (PAGED && zeroed) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(DBAR(B_E + s));
        ++cnt;
      }
      if (!ok) break;
      // ---- merge the four warps' partial states and write this item's partial
      l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
      l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
      l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
      l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
      if (t4 == 0) {
        merge_ml[(warp * 16 + g8) * 2 + 0] = m_lo;
        merge_ml[(warp * 16 + g8) * 2 + 1] = l_lo;
        merge_ml[(warp * 16 + g8 + 8) * 2 + 0] = m_hi;
        merge_ml[(warp * 16 + g8 + 8) * 2 + 1] = l_hi;
      }
      float* mo = merge_o + warp * 16 * C::MC;
#pragma unroll
      for (int pass = 0; pass < D / C::MC; ++pass) {
        // this warp's columns [pass*MC, (pass+1)*MC) of its 16 rows
#pragma unroll
        for (int nn = 0; nn < C::MC / 8; ++nn) {
          const int n = pass * (C::MC / 8) + nn;
          mo[g8 * C::MC + nn * 8 + 2 * t4] = o[n][0];
          mo[g8 * C::MC + nn * 8 + 2 * t4 + 1] = o[n][1];
          mo[(g8 + 8) * C::MC + nn * 8 + 2 * t4] = o[n][2];
          mo[(g8 + 8) * C::MC + nn * 8 + 2 * t4 + 1] = o[n][3];
        }
        mbar_arrive(DBAR(B_M0));
        ok = mbar_wait(DBAR(B_M0), m_cnt & 1u, abort_flag, tmo, ecode | 3);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        for (int idx = threadIdx.x; idx < p.RB * C::MC; idx += 128) {
          const int row = idx / C::MC, dc = idx - row * C::MC;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < 4; ++w) M = fmaxf(M, merge_ml[(w * 16 + row) * 2]);
          float Lsum = 0.f, acc = 0.f;
          if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const float wt = ex2_approx(merge_ml[(w * 16 + row) * 2] - M);
              Lsum += merge_ml[(w * 16 + row) * 2 + 1] * wt;
              acc += merge_o[(w * 16 + row) * C::MC + dc] * wt;
            }
          }
          const int head = hb * p.RB + row;
          const size_t slot = static_cast<size_t>(cid) * p.hq + head;
          const int d = pass * C::MC + dc;
          p.ws_o[slot * D + d] = Lsum > 0.f ? acc / Lsum : 0.f;
          if (d == 0) p.ws_lse[slot] = Lsum > 0.f ? (M + __log2f(Lsum)) * LN2 : -INFINITY;
        }
        mbar_arrive(DBAR(B_M1));
        ok = mbar_wait(DBAR(B_M1), m_cnt & 1u, abort_flag, tmo, ecode | 4);
        ok = __all_sync(0xffffffffu, ok);
        ++m_cnt;
        if (!ok) break;
      }
      ++n_done;
    }
  }
#undef DBAR
  __syncthreads();
}

// Merge kernel: one CTA per (request, KV group); lse = ln sum_c exp(lse_c),
// out = sum_c exp(lse_c - lse) O_c, cast to the output dtype.
template <int D, bool BF16>
__global__ void __launch_bounds__(256)
    mea_lse_merge_kernel(const DecParams p) {
  // One CTA per (request b, KV group g): the R heads of the group, all their chunk partials.
  //   warp w (heads w, w+8, ...): M = max_c lse_c, z = sum_c exp(lse_c - M) -> shared memory;
  //   then thread (head, 4 columns): O = sum_c exp(lse_c - M) O_c / z with float4 loads.
  const int b = blockIdx.x;
  const int g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int s_start;
  __shared__ float s_m[64], s_z[64];
  const int L = __ldg(p.cu_k + b + 1) - __ldg(p.cu_k + b);
  const int n = (L + p.chunk - 1) / p.chunk;
  if (threadIdx.x < 32) {
    const int st = dec_chunk_start(p.cu_k, b, p.chunk);
    if (threadIdx.x == 0) s_start = st;
  }
  __syncthreads();
  const int c0 = s_start;
  using OutT = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  OutT* out = reinterpret_cast<OutT*>(p.out);
  for (int rb = 0; rb < p.R; rb += 64) {  // heads of the group, 64 at a time
    const int rn = min(64, p.R - rb);
    for (int rr = warp; rr < rn; rr += 8) {
      const int head = g * p.R + rb + rr;
      float m = -INFINITY;
      for (int c = lane; c < n; c += 32)
        m = fmaxf(m, p.ws_lse[static_cast<size_t>(c0 + c) * p.hq + head]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      float z = 0.f;
      if (m != -INFINITY)
        for (int c = lane; c < n; c += 32)
          z += __expf(p.ws_lse[static_cast<size_t>(c0 + c) * p.hq + head] - m);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
      if (lane == 0) {
        s_m[rr] = m;
        s_z[rr] = z;
      }
    }
    __syncthreads();
    const int dh4 = p.dh / 4;  // output columns (the partials hold D >= dh)
    for (int idx = threadIdx.x; idx < rn * dh4; idx += blockDim.x) {
      const int rr = idx / dh4, d = (idx - rr * dh4) * 4;
      const int head = g * p.R + rb + rr;
      const float m = s_m[rr], z = s_z[rr];
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m != -INFINITY) {
#pragma unroll 4
        for (int c = 0; c < n; ++c) {
          const size_t slot = static_cast<size_t>(c0 + c) * p.hq + head;
          const float w = __expf(p.ws_lse[slot] - m);
          const float4 o = *reinterpret_cast<const float4*>(p.ws_o + slot * D + d);
          acc.x = fmaf(w, o.x, acc.x);
          acc.y = fmaf(w, o.y, acc.y);
          acc.z = fmaf(w, o.z, acc.z);
          acc.w = fmaf(w, o.w, acc.w);
        }
      }
      const float inv = z > 0.f ? 1.f / z : 0.f;
      OutT* dst = out + (static_cast<size_t>(b) * p.hq + head) * p.dh + d;
      if constexpr (BF16) {
        reinterpret_cast<__nv_bfloat162*>(dst)[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
        reinterpret_cast<__nv_bfloat162*>(dst)[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
      } else {
        reinterpret_cast<__half2*>(dst)[0] = __floats2half2_rn(acc.x * inv, acc.y * inv);
        reinterpret_cast<__half2*>(dst)[1] = __floats2half2_rn(acc.z * inv, acc.w * inv);
      }
      if (d == 0 && p.lse)
        p.lse[static_cast<size_t>(head) * p.n_seqs + b] = z > 0.f ? m + __logf(z) : -INFINITY;
    }
    __syncthreads();
  }
}

}  // namespace mea
