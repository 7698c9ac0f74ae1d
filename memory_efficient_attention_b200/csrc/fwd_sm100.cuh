// fwd_sm100.cuh — persistent, warp-specialised forward kernel of exact attention for sm_100a.
//
// Computes, for every (segment, 128-row query tile, head block), out = softmax(QK^T*scale+bias)V
// and lse, one 128-key tile at a time with an online softmax, so the score matrix only ever
// lives in tensor memory (the blockwise engine of "大模型推理加速终极指南", section 1; masks and
// bias of "How to Build Memory-Efficient Transformers with xFormers…", techniques 1, 3 and 5).
//
// Roles (192 threads, one CTA per SM):
//   warps 0-3  softmax / correction / epilogue: thread r owns row r of the tile = TMEM lane r.
//   warp 4     TMA producer: Q tile once per work item, then K_j, V_j through an NS-slot ring.
//   warp 5     tcgen05 issuer (one lane): S_j = Q K_j^T into TMEM buffer j%2, O += P_j V_j with
//              P_j read from TMEM (written over S_j by the softmax warps). Also owns TMEM.
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D). P_j is bf16/f16-packed in the first 64
// columns of its S buffer.
//
// GQA packing: a 128-row tile holds 128/P tokens x P query heads of one KV group (row r ->
// token tok0 + r/P, head hb*P + r%P), loaded by one 3-D TMA box [128/P tokens, P heads, 64 d],
// so each K/V tile is read once for the P heads that share it.
//
// Work items (tile, segment, head block) are visited round-robin by the persistent CTAs in
// heavy-first order for causal masks (the last query tiles have the most keys).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

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
  int n_hb;          // head blocks = hq / P
  int P;             // query heads packed per tile (a power of two dividing R)
  int R;             // query heads per KV head
  int tok_per_tile;  // 128 / P
  int t_max;         // max query tiles of a segment
  long long n_items; // t_max * n_seqs * n_hb
  float c1;          // scale * log2(e)
  unsigned long long timeout_ns;
};

template <int D>
struct FwdCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int ATOMS = D / 64;  // 128-byte swizzle atoms along the head dim
  static constexpr uint32_t ATOM_BYTES = 128 * 128;
  static constexpr uint32_t TILE_BYTES = 128 * D * 2;
  static constexpr int NS = (D == 128) ? 6 : 8;
  static constexpr uint32_t SMEM_Q = 0;
  static constexpr uint32_t SMEM_KV = TILE_BYTES;
  static constexpr uint32_t SMEM_BAR = SMEM_KV + NS * TILE_BYTES;
  static constexpr uint32_t SMEM_TOTAL = SMEM_BAR + 256 + 1024;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_O = 256;
};

struct FwdItem {
  int seg, hb, q0, lq, k0, lk, tok0, n_kv;
  bool live;
};

__device__ __forceinline__ FwdItem fwd_decode_item(const FwdParams& p, long long lin,
                                                   bool causal) {
  FwdItem it;
  const long long per = static_cast<long long>(p.n_seqs) * p.n_hb;
  const int tr = static_cast<int>(lin / per);
  const int rem = static_cast<int>(lin - static_cast<long long>(tr) * per);
  it.seg = rem / p.n_hb;
  it.hb = rem - it.seg * p.n_hb;
  it.q0 = __ldg(p.cu_q + it.seg);
  it.lq = __ldg(p.cu_q + it.seg + 1) - it.q0;
  it.k0 = __ldg(p.cu_k + it.seg);
  it.lk = __ldg(p.cu_k + it.seg + 1) - it.k0;
  const int nt = (it.lq + p.tok_per_tile - 1) / p.tok_per_tile;
  const int t = causal ? (p.t_max - 1 - tr) : tr;
  it.live = (t >= 0) && (t < nt);
  it.tok0 = t * p.tok_per_tile;
  int kv_end = it.lk;
  if (causal) {
    const int last = min(it.tok0 + p.tok_per_tile, it.lq) - 1;
    kv_end = min(it.lk, last + 1 + it.lk - it.lq);
  }
  it.n_kv = kv_end > 0 ? (kv_end + 127) / 128 : 0;
  return it;
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

template <int D, bool BF16, bool CAUSAL, bool ALIBI>
__global__ void __launch_bounds__(192, 1)
    mea_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_s = sbase + C::SMEM_Q;
  const uint32_t kv_s0 = sbase + C::SMEM_KV;

  constexpr int B_QF = 0, B_QE = 1, B_KVF = 2, B_KVE = 2 + C::NS, B_SF = 2 + 2 * C::NS;
  constexpr int B_PF = B_SF + 2, B_OD = B_PF + 2, B_OE = B_OD + 1, B_DR = B_OE + 1;
  constexpr int N_BARS = B_DR + 1;
  const uint32_t bar0 = sbase + C::SMEM_BAR;
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_BAR + 8 * N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

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
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(B_SF + b), 1);
      mbar_init(BAR(B_PF + b), 128);
    }
    mbar_init(BAR(B_OD), 1);
    mbar_init(BAR(B_OE), 128);
    mbar_init(BAR(B_DR), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t kv_cnt = 0, q_cnt = 0;
      bool ok = true;
      for (long long lin = blockIdx.x; lin < p.n_items && ok; lin += gridDim.x) {
        const FwdItem it = fwd_decode_item(p, lin, CAUSAL);
        if (!it.live || it.n_kv == 0) continue;
        const int g = (it.hb * p.P) / p.R;
        ok = mbar_wait(BAR(B_QE), (q_cnt & 1u) ^ 1u, abort_flag, tmo, ecode | 1);
        if (!ok) break;
        mbar_arrive_expect_tx(BAR(B_QF), C::TILE_BYTES);
#pragma unroll
        for (int a = 0; a < C::ATOMS; ++a)
          tma_load_3d(q_s + a * C::ATOM_BYTES, &tm_q, BAR(B_QF), a * 64, it.hb * p.P,
                      it.q0 + it.tok0);
        ++q_cnt;
        for (int j = 0; j < it.n_kv && ok; ++j) {
#pragma unroll 1
          for (int w = 0; w < 2; ++w) {
            const uint32_t s = kv_cnt % C::NS;
            const uint32_t ph = (kv_cnt / C::NS) & 1u;
            ok = mbar_wait(BAR(B_KVE + s), ph ^ 1u, abort_flag, tmo, ecode | 2);
            if (!ok) break;
            mbar_arrive_expect_tx(BAR(B_KVF + s), C::TILE_BYTES);
            const uint32_t dst = kv_s0 + s * C::TILE_BYTES;
#pragma unroll
            for (int a = 0; a < C::ATOMS; ++a)
              tma_load_3d(dst + a * C::ATOM_BYTES, w ? &tm_v : &tm_k, BAR(B_KVF + s), a * 64, g,
                          it.k0 + j * 128);
            ++kv_cnt;
          }
        }
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
  } else if (warp == 5) {
    // ---------------------------------------------------------------- tcgen05 issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = umma_idesc_f16(BF16, 128, 128, false, false);
      constexpr uint32_t IDESC_PV = umma_idesc_f16(BF16, 128, D, false, true);
      uint32_t kv_cnt = 0, q_cnt = 0, tile = 0, items_pv = 0;
      bool ok = true;
      bool pend_valid = false, pend_first = false;
      uint32_t pend_tile = 0, pend_vslot = 0, pend_vph = 0;

      auto issue_pv = [&]() -> bool {
        const uint32_t b = pend_tile & 1u;
        if (!mbar_wait(BAR(B_PF + b), (pend_tile >> 1) & 1u, abort_flag, tmo, ecode | 3))
          return false;
        if (pend_first) {
          if (!mbar_wait(BAR(B_OE), (items_pv & 1u) ^ 1u, abort_flag, tmo, ecode | 4))
            return false;
          ++items_pv;
        }
        if (!mbar_wait(BAR(B_KVF + pend_vslot), pend_vph, abort_flag, tmo, ecode | 5))
          return false;
        tc_fence_after();
        const uint32_t vbase = kv_s0 + pend_vslot * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint64_t bd = umma_desc_sw128(vbase + kk * 2048, C::ATOM_BYTES, 1024);
          mma_ts(tmem + C::TM_O, tmem + b * 128 + kk * 8, bd, IDESC_PV,
                 (pend_first && kk == 0) ? 0u : 1u);
        }
        mma_commit(BAR(B_KVE + pend_vslot));
        mma_commit(BAR(B_OD));
        return true;
      };

      for (long long lin = blockIdx.x; lin < p.n_items && ok; lin += gridDim.x) {
        const FwdItem it = fwd_decode_item(p, lin, CAUSAL);
        if (!it.live || it.n_kv == 0) continue;
        ok = mbar_wait(BAR(B_QF), q_cnt & 1u, abort_flag, tmo, ecode | 6);
        if (!ok) break;
        tc_fence_after();
        for (int j = 0; j < it.n_kv; ++j) {
          const uint32_t s = kv_cnt % C::NS;
          const uint32_t ph = (kv_cnt / C::NS) & 1u;
          ok = mbar_wait(BAR(B_KVF + s), ph, abort_flag, tmo, ecode | 7);
          if (!ok) break;
          tc_fence_after();
          const uint32_t b = tile & 1u;
          const uint32_t kbase = kv_s0 + s * C::TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
            const uint64_t ad = umma_desc_sw128(q_s + off, 16, 1024);
            const uint64_t bd = umma_desc_sw128(kbase + off, 16, 1024);
            mma_ss(tmem + b * 128, ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
          }
          mma_commit(BAR(B_SF + b));
          mma_commit(BAR(B_KVE + s));
          if (j == it.n_kv - 1) mma_commit(BAR(B_QE));
          ++kv_cnt;
          const uint32_t vs = kv_cnt % C::NS;
          const uint32_t vph = (kv_cnt / C::NS) & 1u;
          ++kv_cnt;
          if (pend_valid) {
            ok = issue_pv();
            if (!ok) break;
          }
          pend_valid = true;
          pend_first = (j == 0);
          pend_tile = tile;
          pend_vslot = vs;
          pend_vph = vph;
          ++tile;
        }
        if (!ok) break;
        ++q_cnt;
      }
      if (ok && pend_valid) ok = issue_pv();
      // Every MMA issued so far must finish before TMEM is released.
      mma_commit(BAR(B_DR));
      volatile int never = 0;
      mbar_wait(BAR(B_DR), 0, &never, tmo, ecode | 14);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps 0-3
    const int r = threadIdx.x;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    constexpr float LOG2E = 1.4426950408889634f;
    constexpr float LN2 = 0.6931471805599453f;
    uint32_t tile = 0;
    bool ok = true;
    for (long long lin = blockIdx.x; lin < p.n_items && ok; lin += gridDim.x) {
      const FwdItem it = fwd_decode_item(p, lin, CAUSAL);
      if (!it.live) continue;
      const int tok = it.tok0 + r / p.P;
      const int head = it.hb * p.P + (r % p.P);
      const bool row_valid = tok < it.lq;
      using OutT = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
      OutT* orow = reinterpret_cast<OutT*>(p.out) +
                   (static_cast<size_t>(it.q0 + tok) * p.hq + head) * D;
      if (it.n_kv == 0) {
        if (row_valid) {
          uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int i = 0; i < D / 8; ++i) reinterpret_cast<uint4*>(orow)[i] = z;
          if (p.lse) p.lse[static_cast<size_t>(head) * p.total_q + it.q0 + tok] = -INFINITY;
        }
        continue;
      }
      const int pos = tok + it.lk - it.lq;       // key position of this query row
      const int p_min = it.tok0 + it.lk - it.lq;  // position of the tile's first row
      float slope2 = 0.f;
      if constexpr (ALIBI) slope2 = __ldg(p.slopes + head) * LOG2E;
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < it.n_kv; ++j) {
        const uint32_t b = tile & 1u;
        ok = mbar_wait(BAR(B_SF + b), (tile >> 1) & 1u, abort_flag, tmo, ecode | 8);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[128];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          tmem_ld32(t_lane + b * 128 + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c4 * 32]));
        tmem_wait_ld();
        const int kv0 = j * 128;
        const bool need_mask = (kv0 + 128 > it.lk) || (CAUSAL && kv0 + 127 > p_min);
        const int limit = (CAUSAL ? min(pos, it.lk - 1) : it.lk - 1) - kv0;
        const float dd0 = static_cast<float>(kv0 - pos);
        float x[128];
        float mt = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          float v = __uint_as_float(sr[c]) * p.c1;
          if constexpr (ALIBI) v = fmaf(-slope2, fabsf(dd0 + static_cast<float>(c)), v);
          if (need_mask && c > limit) v = -INFINITY;
          x[c] = v;
          mt = fmaxf(mt, v);
        }
        const float m_new = fmaxf(m_ref, mt);
        const bool resc = m_new > m_ref + 8.0f;
        float alpha = 1.f;
        if (resc) {
          alpha = ex2_approx(m_ref - m_new);
          l *= alpha;
          m_ref = m_new;
        }
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        float rs = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = ex2_approx(x[c4 * 32 + 2 * i] - m_use);
            const float p1 = ex2_approx(x[c4 * 32 + 2 * i + 1] - m_use);
            rs += p0 + p1;
            pk[i] = pack2<BF16>(p0, p1);
          }
          tmem_st16(t_lane + b * 128 + c4 * 16, pk);
        }
        l += rs;
        tmem_wait_st();
        if (j > 0) {
          // O += P_{j-1} V_{j-1} must be complete before O is rescaled (and is waited on once
          // per tile in order, so the barrier phases are never skipped).
          ok = mbar_wait(BAR(B_OD), (tile - 1) & 1u, abort_flag, tmo, ecode | 9);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          if (__any_sync(0xffffffffu, resc)) {
            tc_fence_after();
#pragma unroll 1
            for (int c4 = 0; c4 < D / 32; ++c4) {
              uint32_t o[32];
              tmem_ld32(t_lane + C::TM_O + c4 * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(t_lane + C::TM_O + c4 * 32, o);
            }
            tmem_wait_st();
          }
        }
        tc_fence_before();
        mbar_arrive(BAR(B_PF + b));
        ++tile;
      }
      if (!ok) break;
      // ---- epilogue: O / l -> out, lse
      ok = mbar_wait(BAR(B_OD), (tile - 1) & 1u, abort_flag, tmo, ecode | 10);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c4 = 0; c4 < D / 32; ++c4) {
        uint32_t o[32];
        tmem_ld32(t_lane + C::TM_O + c4 * 32, o);
        tmem_wait_ld();
        if (row_valid) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv_l,
                                __uint_as_float(o[2 * i + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(BAR(B_OE));
      if (row_valid && p.lse)
        p.lse[static_cast<size_t>(head) * p.total_q + it.q0 + tok] =
            l > 0.f ? (m_ref + __log2f(l)) * LN2 : -INFINITY;
    }
  }
#undef BAR
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace mea
