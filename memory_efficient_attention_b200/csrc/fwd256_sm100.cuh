// fwd256_sm100.cuh — forward kernel of exact attention for head dims 136..256 (sm_100a).
//
// The same computation as mea_fwd_sm100_kernel (online softmax over 128-key tiles; masks, GQA
// packing and ALiBi of "How to Build Memory-Efficient Transformers with xFormers…", techniques
// 1, 3 and 5), laid out for a 256-wide head: O of one 128-row query tile already takes half of
// the 512 tensor-memory columns, so a work item is ONE sub-tile, and the two remaining 128-column
// regions double-buffer S. Q·Kᵀ of tile t+1 then runs while the softmax works on tile t, and the
// tensor core alternates P·V(t), Q·Kᵀ(t+2) with no wait on its own results.
//
// Roles (384 threads, one CTA per SM; warps 10-11 only lend their registers):
//   warps 0-3  softmax of the sub-tile (thread r = row r = TMEM lane r); rescale of O when the
//              running maximum moves by more than 2^8.
//   warps 4-7  epilogue: O / l -> out and lse once the item's last P·V has finished, so the
//              softmax warps go straight on to the next item.
//   warp 8     tcgen05 issuer (one lane); owns TMEM.
//   warp 9     scheduler and TMA producer (the live-item walk of the 128-wide kernel).
// TMEM columns: S_0 [0,128), S_1 [128,256), O [256,512). P(t) is written bf16/f16-packed over
// the first 64 columns of its S buffer.
// Shared memory: Q (128 rows x 256 columns, four 128-byte swizzle atoms) and a ring of five
// 32 KB half tiles (128 keys x 128 columns): a K or V tile is two halves, loaded in the order
// K(0), K(1), V(0), K(2), V(1), K(3), ... in which the issuer uses them.
#pragma once

#include "fwd_sm100.cuh"

namespace mea {

struct Fwd256Cfg {
  static constexpr int D = 256;
  static constexpr int ATOMS = 4;                        // 64-column atoms along D
  static constexpr uint32_t ATOM_BYTES = 128 * 128;      // 128 rows x 128 bytes
  static constexpr uint32_t Q_BYTES = ATOMS * ATOM_BYTES;
  static constexpr uint32_t HALF_BYTES = 2 * ATOM_BYTES; // 128 keys x 128 columns
  static constexpr int NS = 5;                           // half-tile ring slots
  static constexpr int QD = 4;                           // work-item queue depth
  static constexpr int MAXSEG = 64;                      // segments ranked in shared memory
  static constexpr uint32_t SMEM_Q = 0;
  static constexpr uint32_t SMEM_KV = Q_BYTES;
  static constexpr uint32_t SMEM_MISC = SMEM_KV + NS * HALF_BYTES;  // barriers, TMEM slot, queue
  static constexpr uint32_t MISC_BYTES = 512;
  static constexpr uint32_t MISC_QUEUE = 320;
  static constexpr uint32_t SMEM_STATS = SMEM_MISC + MISC_BYTES;  // m, l of the 128 rows
  static constexpr uint32_t SMEM_SEG = SMEM_STATS + 128 * 8;
  static constexpr uint32_t SMEM_TOTAL = SMEM_SEG + MAXSEG * 6 + 1024;
  static_assert(SMEM_TOTAL <= 232448, "shared memory per CTA");
  static_assert(MISC_QUEUE + QD * 32 <= MISC_BYTES, "queue region");
  static constexpr int THREADS = 384;
  static constexpr int REGS_SOFTMAX = 208;               // warps 0-7
  static constexpr int REGS_OTHER = 80;                  // warps 8-11
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_O = 256;
};

template <bool BF16, bool CAUSAL, bool ALIBI>
__global__ void __launch_bounds__(384, 1)
    mea_fwd256_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = Fwd256Cfg;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_s = sbase + C::SMEM_Q;
  const uint32_t kv_s0 = sbase + C::SMEM_KV;

  constexpr int B_QF = 0, B_QE = 1, B_KVF = 2, B_KVE = 2 + C::NS, B_SF = 2 + 2 * C::NS;
  constexpr int B_PF = B_SF + 2, B_OR = B_PF + 2, B_OF = B_OR + 1, B_OE = B_OF + 1;
  constexpr int B_STF = B_OE + 1, B_STE = B_STF + 1, B_DR = B_STE + 1;
  constexpr int B_IF = B_DR + 1, B_IE = B_IF + C::QD;
  constexpr int N_BARS = B_IE + C::QD;
  static_assert(8 * N_BARS + 8 <= C::MISC_QUEUE, "barrier region");
  const uint32_t bar0 = sbase + C::SMEM_MISC;
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC + 8 * N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t queue = sbase + C::SMEM_MISC + C::MISC_QUEUE;
  float* stats = reinterpret_cast<float*>(smem + C::SMEM_STATS);  // m[128], then l[128]
  const uint32_t s_np = sbase + C::SMEM_SEG;
  const uint32_t s_id = s_np + 4u * C::MAXSEG;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t tmo = p.timeout_ns;
  const unsigned ecode = KID_FWD << 8 | 0x40;

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_QF), 1);
    mbar_init(BAR(B_QE), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(BAR(B_KVF + s), 1);
      mbar_init(BAR(B_KVE + s), 1);
    }
    mbar_init(BAR(B_SF), 1);
    mbar_init(BAR(B_SF + 1), 1);
    // P of the tile in S buffer b: one elected arrival per softmax warp. One barrier per
    // buffer: S(t+1) is ready before P(t) is consumed, so a warp can finish tile t+1 while
    // another is still on tile t, and its arrival must not count towards tile t.
    mbar_init(BAR(B_PF), 4);
    mbar_init(BAR(B_PF + 1), 4);
    mbar_init(BAR(B_OR), 1);
    mbar_init(BAR(B_OF), 1);
    mbar_init(BAR(B_OE), 128);   // every epilogue thread
    mbar_init(BAR(B_STF), 128);  // every softmax thread
    mbar_init(BAR(B_STE), 128);  // every epilogue thread
    mbar_init(BAR(B_DR), 1);
    for (int s = 0; s < C::QD; ++s) {
      mbar_init(BAR(B_IF + s), 1);
      mbar_init(BAR(B_IE + s), 9);  // the issuer and one elected lane per softmax/epilogue warp
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  // Segment ranking, as in the 128-wide kernel (the K/V ring is the scratch area: nothing is
  // loaded into it before the barrier below).
  const bool ranked = p.n_seqs <= C::MAXSEG;
  if (ranked) {
    const uint32_t tmp = kv_s0;
    for (int s = threadIdx.x; s < p.n_seqs; s += blockDim.x)
      sts_s32(tmp + 4u * s, fwd_seg_pairs(p, s));
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
    // The scratch counts sat in the K/V ring, which the TMA (async proxy) writes next.
    fence_proxy_async_smem();
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
      FwdWalk w;
      fwd_walk_init(p, w, ranked, s_np);
      int seg = 0, pair = 0, hb = 0;
      bool have = fwd_walk_next(p, w, ranked, s_np, s_id, seg, pair, hb);
      FwdItem cur{};
      if (have) cur = fwd_make_item(p, seg, pair, hb, CAUSAL);
      // One K or V tile = two half tiles (columns [0,128) and [128,256)) in consecutive slots.
      auto load_tile = [&](const CUtensorMap* map, int key0, int g) {
#pragma unroll 1
        for (int half = 0; half < 2 && ok; ++half) {
          const uint32_t s = kv_cnt % C::NS;
          ok = mbar_wait(BAR(B_KVE + s), ((kv_cnt / C::NS) & 1u) ^ 1u, abort_flag, tmo, ecode | 2);
          if (!ok) break;
          mbar_arrive_expect_tx(BAR(B_KVF + s), C::HALF_BYTES);
          const uint32_t dst = kv_s0 + s * C::HALF_BYTES;
          tma_load_3d(dst, map, BAR(B_KVF + s), (2 * half) * 64, g, key0);
          tma_load_3d(dst + C::ATOM_BYTES, map, BAR(B_KVF + s), (2 * half + 1) * 64, g, key0);
          ++kv_cnt;
        }
      };
      while (ok) {
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
        const int n = cur.n_kv0;
        if (n > 0) {
          const int g = fwd_group_of(p, cur.hb);
          ok = mbar_wait(BAR(B_QE), (q_cnt & 1u) ^ 1u, abort_flag, tmo, ecode | 1);
          if (!ok) break;
          mbar_arrive_expect_tx(BAR(B_QF), C::Q_BYTES);
#pragma unroll
          for (int a = 0; a < C::ATOMS; ++a)
            tma_load_3d(q_s + a * C::ATOM_BYTES, &tm_q, BAR(B_QF), a * 64, cur.hb << p.log2_p,
                        cur.q0 + cur.tok0);
          ++q_cnt;
          // Step t of the issuer visits key tile n-1-t (diagonal first).
          load_tile(&tm_k, cur.k0 + (n - 1) * 128, g);
          if (n > 1) load_tile(&tm_k, cur.k0 + (n - 2) * 128, g);
          for (int t = 0; t < n && ok; ++t) {
            load_tile(&tm_v, cur.k0 + (n - 1 - t) * 128, g);
            if (t + 2 < n) load_tile(&tm_k, cur.k0 + (n - 3 - t) * 128, g);
          }
          const int nm = nxt.n_kv0;
          if (ok && have2 && nm > 0) {
            const int ng = fwd_group_of(p, nxt.hb);
#pragma unroll
            for (int a = 0; a < C::ATOMS; ++a) {
              tma_prefetch_l2_3d(&tm_q, a * 64, nxt.hb << p.log2_p, nxt.q0 + nxt.tok0);
              tma_prefetch_l2_3d(&tm_k, a * 64, ng, nxt.k0 + (nm - 1) * 128);
            }
          }
        }
        cur = nxt;
        have = have2;
      }
      if (!ok) {
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
      constexpr uint32_t IDESC_QK = umma_idesc_f16(BF16, 128, 128, false, false);
      constexpr uint32_t IDESC_PV = umma_idesc_f16(BF16, 128, 128, false, true);
      uint32_t kv_cnt = 0, q_cnt = 0, it_cnt = 0, oe_cnt = 0, g = 0;
      bool ok = true;
      // Waits for the two half tiles of the next K or V tile; returns the slot of the first.
      auto take_tile = [&](uint32_t& s0, uint32_t& s1) {
        s0 = kv_cnt % C::NS;
        s1 = (kv_cnt + 1) % C::NS;
        ok = ok && mbar_wait(BAR(B_KVF + s0), (kv_cnt / C::NS) & 1u, abort_flag, tmo, ecode | 7);
        ok = ok && mbar_wait(BAR(B_KVF + s1), ((kv_cnt + 1) / C::NS) & 1u, abort_flag, tmo,
                             ecode | 7);
        kv_cnt += 2;
        tc_fence_after();
      };
      while (ok) {
        const uint32_t slot = it_cnt % C::QD;
        ok = mbar_wait(BAR(B_IF + slot), (it_cnt / C::QD) & 1u, abort_flag, tmo, ecode | 13);
        if (!ok) break;
        const FwdItem it = fwd_read_item(queue + 32u * slot);
        mbar_arrive(BAR(B_IE + slot));
        ++it_cnt;
        if (it.hb < 0) break;
        const int n = it.n_kv0;
        if (n == 0) continue;
        ok = mbar_wait(BAR(B_QF), q_cnt & 1u, abort_flag, tmo, ecode | 6);
        if (!ok) break;
        tc_fence_after();
        // ---- S(t) = Q K(t)^T into buffer (g + t) % 2
        auto issue_qk = [&](int t) {
          uint32_t s0, s1;
          take_tile(s0, s1);
          if (!ok) return;
          const uint32_t b = (g + t) & 1u;
#pragma unroll
          for (int kk = 0; kk < C::D / 16; ++kk) {
            const int a = kk >> 2;
            const uint32_t koff = (a & 1) * C::ATOM_BYTES + (kk & 3) * 32;
            const uint64_t ad = umma_desc_sw128(q_s + a * C::ATOM_BYTES + (kk & 3) * 32, 16, 1024);
            const uint64_t bd =
                umma_desc_sw128(kv_s0 + ((a >> 1) ? s1 : s0) * C::HALF_BYTES + koff, 16, 1024);
            mma_ss(tmem + b * 128, ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
          }
          mma_commit(BAR(B_SF + b));
          mma_commit(BAR(B_KVE + s0));
          mma_commit(BAR(B_KVE + s1));
          if (t == n - 1) mma_commit(BAR(B_QE));
        };
        // ---- O += P(t) V(t), columns [0,128) from the first half tile, [128,256) the second
        auto issue_pv = [&](int t) {
          const uint32_t gt = g + static_cast<uint32_t>(t);
          ok = ok && mbar_wait_spin(BAR(B_PF + (gt & 1u)), (gt >> 1) & 1u, abort_flag, tmo,
                                    ecode | 3);
          if (ok && t == 0) {
            ok = mbar_wait(BAR(B_OE), (oe_cnt & 1u) ^ 1u, abort_flag, tmo, ecode | 4);
            ++oe_cnt;
          }
          uint32_t s0, s1;
          take_tile(s0, s1);
          if (!ok) return;
          const uint32_t b = (g + t) & 1u;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint32_t vbase = kv_s0 + (half ? s1 : s0) * C::HALF_BYTES;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t bd = umma_desc_sw128(vbase + kk * 16 * 128, C::ATOM_BYTES, 1024);
              mma_ts(tmem + C::TM_O + half * 128, tmem + b * 128 + kk * 8, bd, IDESC_PV,
                     (t == 0 && kk == 0) ? 0u : 1u);
            }
          }
          mma_commit(BAR(B_OR));
          mma_commit(BAR(B_KVE + s0));
          mma_commit(BAR(B_KVE + s1));
          if (t == n - 1) mma_commit(BAR(B_OF));
        };
        issue_qk(0);
        if (n > 1) issue_qk(1);
        for (int t = 0; t < n && ok; ++t) {
          issue_pv(t);
          if (t + 2 < n) issue_qk(t + 2);
        }
        if (!ok) break;
        g += static_cast<uint32_t>(n);
        ++q_cnt;
      }
      mma_commit(BAR(B_DR));
      volatile int never = 0;
      mbar_wait(BAR(B_DR), 0, &never, tmo, ecode | 14);
    }
    }
    fwd_teardown(warp == 8, tmem, C::TMEM_COLS);
  } else if (warp < 4) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
    // ---------------------------------------------------------------- softmax warpgroup
    const int r = threadIdx.x;  // row = TMEM lane
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t t_o = t_lane + C::TM_O;
    constexpr float LOG2E = 1.4426950408889634f;
    uint32_t it_cnt = 0, g = 0, st_cnt = 0;
    bool ok = true;
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
      const int n = it.n_kv0;
      if (n == 0) continue;
      const int tok = it.tok0 + (r >> p.log2_p);
      const int head = (it.hb << p.log2_p) + (r & (p.P - 1));
      const int pos = tok + it.lk - it.lq;
      const int p_min = it.tok0 + it.lk - it.lq;
      float slope2 = 0.f;
      if constexpr (ALIBI) slope2 = __ldg(p.slopes + head) * LOG2E;
      float m_ref = -INFINITY, l = 0.f;
      for (int jj = 0; jj < n; ++jj) {
        const uint32_t gt = g + static_cast<uint32_t>(jj);
        const uint32_t b = gt & 1u;
        ok = mbar_wait(BAR(B_SF + b), (gt >> 1) & 1u, abort_flag, tmo, ecode | 8);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float alpha = 1.f;
        const bool resc = fwd_softmax_tile<BF16, CAUSAL, ALIBI, false, true>(
            p, t_lane + b * 128, (n - 1 - jj) * 128, it.lk, pos, p_min, slope2, m_ref, l, alpha);
        if (jj > 0 && __any_sync(0xffffffffu, resc)) {
          // O holds the tiles before this one once the previous P·V has finished.
          ok = mbar_wait(BAR(B_OR), (gt - 1) & 1u, abort_flag, tmo, ecode | 9);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c4 = 0; c4 < C::D / 32; ++c4) {
            uint32_t o[32];
            tmem_ld32(t_o + c4 * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(t_o + c4 * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_PF + b));
      }
      if (!ok) break;
      g += static_cast<uint32_t>(n);
      // Hand m and l of this row to the epilogue warps.
      ok = mbar_wait(BAR(B_STE), (st_cnt & 1u) ^ 1u, abort_flag, tmo, ecode | 10);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      stats[r] = m_ref;
      stats[128 + r] = l;
      mbar_arrive(BAR(B_STF));
      ++st_cnt;
    }
    fwd_teardown(false, tmem, C::TMEM_COLS);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
    // ---------------------------------------------------------------- epilogue warpgroup
    const int r = threadIdx.x - 128;  // row = TMEM lane
    const uint32_t t_o = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + C::TM_O;
    constexpr float LN2 = 0.6931471805599453f;
    using OutT = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    const bool out_al32 = (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0 && (p.dh & 15) == 0;
    uint32_t it_cnt = 0, ocnt = 0, st_cnt = 0;
    bool ok = true;
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
      const int tok = it.tok0 + (r >> p.log2_p);
      const int head = (it.hb << p.log2_p) + (r & (p.P - 1));
      const bool row_valid = tok < it.lq;
      OutT* orow = reinterpret_cast<OutT*>(p.out) +
                   (static_cast<size_t>(it.q0 + tok) * p.hq + head) * p.dh;
      float* lse_at = p.lse ? p.lse + static_cast<size_t>(head) * p.total_q + it.q0 + tok : nullptr;
      if (it.n_kv0 == 0) {
        if (row_valid) {
          for (int i = 0; i < (p.dh >> 3); ++i)
            reinterpret_cast<uint4*>(orow)[i] = make_uint4(0, 0, 0, 0);
          if (lse_at) *lse_at = -INFINITY;
        }
        continue;
      }
      ok = mbar_wait(BAR(B_OF), ocnt & 1u, abort_flag, tmo, ecode | 5);
      ok = ok && mbar_wait(BAR(B_STF), st_cnt & 1u, abort_flag, tmo, ecode | 10);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++ocnt;
      tc_fence_after();
      const float m = stats[r], l = stats[128 + r];
      mbar_arrive(BAR(B_STE));
      ++st_cnt;
      const float inv_l = l > 0.f ? p.o_scale / l : 0.f;
      // The row of O in 32-column pieces, packed as it arrives; then O is free for the next
      // item's first P·V.
      uint32_t o[C::D / 2];
#pragma unroll
      for (int c4 = 0; c4 < C::D / 32; ++c4) {
        uint32_t x[32];
        tmem_ld32(t_o + c4 * 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          o[c4 * 16 + i] = pack2<BF16>(__uint_as_float(x[2 * i]) * inv_l,
                                       __uint_as_float(x[2 * i + 1]) * inv_l);
      }
      tc_fence_before();
      mbar_arrive(BAR(B_OE));
      if (row_valid) {
        if (lse_at) *lse_at = l > 0.f ? (m + __log2f(l)) * LN2 : -INFINITY;
        if (out_al32) {
#pragma unroll
          for (int i = 0; i < C::D / 16; ++i)
            if (i < (p.dh >> 4)) st_global_v8(orow + i * 16, &o[8 * i]);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
          for (int i = 0; i < C::D / 8; ++i)
            if (i < (p.dh >> 3))
              dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
      }
    }
    fwd_teardown(false, tmem, C::TMEM_COLS);
  }
#undef BAR
}

}  // namespace mea
