// bwd_tc_sm100.cuh — backward pass of exact attention on the sm_100a tensor cores (tcgen05).
//
// Same definition as the forward (packed varlen, block-diagonal, bottom-right causal, GQA,
// ALiBi); the gradients are the calculus of the forward:
//   P = exp(S - lse),  dS = P * (dO V^T - delta)  with delta = rowsum(dO * O),
//   dV_g += P^T dO,  dK_g += scale * dS^T Q,  dQ = scale * dS K.
// ("How to Build Memory-Efficient Transformers with xFormers…", section "效能對比" times the
// forward and backward of this attention; it prints no formula.)
//
// mea_bwd_dkdv_tc_kernel: one CTA per (128-key tile, segment, KV head). For every query tile of
// the R heads of the group that sees the key tile:
//   S^T = K Q^T, dP^T = V dO^T      (tcgen05, K-major operands, fp32 in TMEM)
//   P^T, dS^T                        (elementwise warpgroup: thread = key = TMEM lane); dS^T
//                                    16-bit-packed over the first 64 columns of dP^T, P^T into
//                                    shared memory as a K-major operand
//   dK += dS^T Q, dV += P^T dO       (tcgen05; A from TMEM / shared memory, B = the [rows][D]
//                                    tiles MN-major)
// TMEM: S^T [0,128), dP^T [128,256), dV [256,256+D), dK [256+D,256+2D). dK and dV accumulate
// over the whole GQA group; they are written once. Since P^T does not sit in TMEM, S^T(i+1) is
// computed while the elementwise warps still work on iteration i.
//
// mea_bwd_dq_tc_kernel: one CTA per (128-row query tile, segment, group of mq query heads);
// for each head in turn (an item), over the key tiles the rows see: S = Q K^T, dP = dO V^T, dS
// (thread = row), dQ += dS K. TMEM: S(j) in [0,128) or [128,256) by the parity of j (counted over
// the CTA's items), dP [256,384), dQ [384,384+D); S(j+2) is computed while the elementwise warps
// work on tile j+1, and the next item's Q/dO load and first S/dP overlap the current item's last
// tile and the read-out of its dQ.
//
// Roles (NWG*128 + 64 threads): NWG elementwise warpgroups (thread = TMEM lane; group w handles
// the 32-column chunks [128w/NWG, 128(w+1)/NWG) of the S/dP tiles and writes its packed P / dS
// over the first half of its own columns, so the groups never touch each other's columns), warp
// 4*NWG the tcgen05 issuer (owns TMEM), warp 4*NWG+1 the TMA producer. Every wait is bounded (all
// hand-offs are mbarriers); no named barriers in the role loops.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "bwd_sm100.cuh"
#include "ptx.cuh"

namespace mea {

template <int D>
struct BwdTcCfg {
  static constexpr int ATOMS = D / 64;
  static constexpr uint32_t ATOM_BYTES = 128 * 128;      // 128 rows x 128 B
  static constexpr uint32_t TILE_BYTES = 128 * D * 2;
  static constexpr int NWG = 4;                          // elementwise warpgroups
  static constexpr int CPW = 4 / NWG;                      // 32-column chunks per group
  static constexpr int THREADS = NWG * 128 + 64;
  static constexpr int W_ISSUE = 4 * NWG, W_LOAD = 4 * NWG + 1;
  // Column of the packed 16-bit operand for 16-row step k16 of a 128-column tile: chunk k16/2
  // (32 rows) was packed by its group at the start of the chunk's own 32 columns... precisely,
  // group w packs its chunks contiguously from column 32*CPW*w.
  __device__ static constexpr uint32_t packed_col(int k16) {
    return static_cast<uint32_t>(32 * CPW * ((k16 >> 1) / CPW) + ((k16 >> 1) % CPW) * 16 +
                                 (k16 & 1) * 8);
  }
  static constexpr uint32_t TMEM_COLS = 512;
};

template <bool BF16>
__device__ __forceinline__ uint32_t bpack2(float lo, float hi) {
  return dpack2<BF16>(lo, hi);
}

// Bias forms of the scores: none, causal ALiBi (the distance row + shift - key is >= 0 wherever
// p can be non-zero, so the bias is linear in row and key), ALiBi without the causal mask
// (|row + shift - key|).
enum { BIAS_NONE = 0, BIAS_LINEAR = 1, BIAS_ABS = 2 };

// dK/dV elementwise step, phase A, for a 32-row chunk of S^T and this thread's key:
//   p_e = 2^(c1 S_e + na_e + kb),  e = 0..31 (row rc0 + e)
// with na_e the row's exponent term from the pre kernel (-lse log2 e; causal ALiBi also
// - slope2 e) read at na_row[e] (the same address in every lane: one broadcast load), kb this
// thread's key term (BIAS_LINEAR: -slope2 (rc0 + shift - key)); BIAS_ABS subtracts
// slope2 |dabs + e| per element. MASK: p_e = 0 outside e_lo <= e < e_hi. Pairs of columns go
// through the f32x2 pipe.
template <bool MASK, int BIAS>
__device__ __forceinline__ void bwd_kv_p(const uint32_t (&sv)[32], const float* na_row,
                                         uint64_t c1x2, uint64_t kb2, float slope2, float dabs,
                                         int e_lo, int e_hi, float (&pr)[32]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    uint64_t b2 = f2_pack(__ldg(na_row + 2 * j), __ldg(na_row + 2 * j + 1));
    if constexpr (BIAS == BIAS_LINEAR) b2 = f2_add(b2, kb2);
    const uint64_t z2 =
        f2_fma(f2_pack(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1])), c1x2, b2);
    float z0, z1;
    f2_unpack(z2, z0, z1);
    if constexpr (BIAS == BIAS_ABS) {
      z0 = fmaf(-slope2, fabsf(dabs + static_cast<float>(2 * j)), z0);
      z1 = fmaf(-slope2, fabsf(dabs + static_cast<float>(2 * j + 1)), z1);
    }
    float p0 = ex2_approx(z0), p1 = ex2_approx(z1);
    if constexpr (MASK) {
      p0 = (2 * j >= e_lo && 2 * j < e_hi) ? p0 : 0.f;
      p1 = (2 * j + 1 >= e_lo && 2 * j + 1 < e_hi) ? p1 : 0.f;
    }
    pr[2 * j] = p0;
    pr[2 * j + 1] = p1;
  }
}

// Phase B for half H (rows 16H .. 16H+15 of the chunk): dS_e = p_e (dP_e + nd_e) with
// nd_e = -delta_e from the pre kernel (broadcast loads at nd_row[e]); dv holds the half's 16
// dP^T columns; dS comes out packed to 16 bits, eight words.
template <bool BF16, int H>
__device__ __forceinline__ void bwd_kv_ds(const float (&pr)[32], const uint32_t (&dv)[16],
                                          const float* nd_row, uint32_t (&pd)[8]) {
#pragma unroll
  for (int jj = 0; jj < 8; ++jj) {
    const int j = H * 8 + jj;
    const uint64_t d2 = f2_mul(
        f2_pack(pr[2 * j], pr[2 * j + 1]),
        f2_add(f2_pack(__uint_as_float(dv[2 * jj]), __uint_as_float(dv[2 * jj + 1])),
               f2_pack(__ldg(nd_row + 2 * j), __ldg(nd_row + 2 * j + 1))));
    float d0, d1;
    f2_unpack(d2, d0, d1);
    pd[jj] = bpack2<BF16>(d0, d1);
  }
}

// dQ elementwise step for one 32-key chunk of the S / dP tiles and this thread's row:
//   p_e = 2^(c1 S_e + b + slope2 e),  dS_e = p_e (dP_e - delta),  e = 0..31 (key kc0 + e)
// with b = -lse log2 e (BIAS_LINEAR: - slope2 (row + shift - kc0)); BIAS_ABS subtracts
// slope2 |dabs - e| per element (dabs = row + shift - kc0). MASK: p_e = 0 for e >= e_hi. dS
// leaves packed to 16 bits, eight words at a time, to TMEM at t_d.
template <bool BF16, bool MASK, int BIAS>
__device__ __forceinline__ void bwd_q_chunk(const uint32_t (&sv)[32], const uint32_t (&dv)[32],
                                            uint64_t c1x2, float b, float slope2, float dabs,
                                            uint64_t nd2, int e_hi, uint32_t t_d) {
  const uint64_t b2 = f2_pack(b, b);
  const uint64_t s2 = f2_pack(slope2, slope2);
  const uint64_t two2 = f2_pack(2.f, 2.f);
  uint64_t e2 = f2_pack(0.f, 1.f);  // exact small integers
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
  uint32_t pd[8];
#pragma unroll
  for (int jj = 0; jj < 8; ++jj) {
    const int j = hh * 8 + jj;
    uint64_t t2 = b2;
    if constexpr (BIAS == BIAS_LINEAR) {
      t2 = f2_fma(s2, e2, b2);
      e2 = f2_add(e2, two2);
    }
    const uint64_t z2 =
        f2_fma(f2_pack(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1])), c1x2, t2);
    float z0, z1;
    f2_unpack(z2, z0, z1);
    if constexpr (BIAS == BIAS_ABS) {
      z0 = fmaf(-slope2, fabsf(dabs - static_cast<float>(2 * j)), z0);
      z1 = fmaf(-slope2, fabsf(dabs - static_cast<float>(2 * j + 1)), z1);
    }
    float p0 = ex2_approx(z0), p1 = ex2_approx(z1);
    if constexpr (MASK) {
      p0 = 2 * j < e_hi ? p0 : 0.f;
      p1 = 2 * j + 1 < e_hi ? p1 : 0.f;
    }
    const uint64_t d2 = f2_mul(
        f2_pack(p0, p1),
        f2_add(f2_pack(__uint_as_float(dv[2 * j]), __uint_as_float(dv[2 * j + 1])), nd2));
    float d0, d1;
    f2_unpack(d2, d0, d1);
    pd[jj] = bpack2<BF16>(d0, d1);
  }
  tmem_st8(t_d + hh * 8, pd);
  }
}

// -------------------------------------------------------------------------------------------
// dK/dV kernel layout: K and V loaded once; Q and dO in a 2-stage ring; P^T (128 keys x 128
// query rows, 16-bit) written by the elementwise warps as the K-major, 128-byte-swizzled A
// operand of dV += P^T dO.
template <int D>
struct BwdKvCfg {
  using T = BwdTcCfg<D>;
  static constexpr uint32_t SMEM_K = 0, SMEM_V = T::TILE_BYTES;
  static constexpr uint32_t SMEM_RING = 2 * T::TILE_BYTES;  // 2 stages x (Q, dO)
  static constexpr uint32_t SMEM_PT = 6 * T::TILE_BYTES;    // 2 atoms of 128 rows x 128 B
  static constexpr uint32_t SMEM_BAR = SMEM_PT + 2 * T::ATOM_BYTES;
  static constexpr uint32_t SMEM_TOTAL = SMEM_BAR + 256 + 1024;
  static_assert(SMEM_TOTAL <= 232448, "shared memory per CTA");
};

template <int D, bool BF16, bool CAUSAL, bool ALIBI>
__global__ void __launch_bounds__(BwdTcCfg<D>::THREADS, 1)
    mea_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_do,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const BwdParams p,
                           unsigned long long timeout_ns) {
  using C = BwdTcCfg<D>;
  using L = BwdKvCfg<D>;
  static_assert(C::NWG == 4, "one 32-row chunk per elementwise warpgroup");
  constexpr float LOG2E = 1.4426950408889634f;
  // segments in decreasing order of work (the pre kernel's ranking), key tiles heaviest first
  const int jt = blockIdx.x, s = p.order ? p.order[blockIdx.y] : blockIdx.y, g = blockIdx.z;
  const int q0 = __ldg(p.cu_q + s), lq = __ldg(p.cu_q + s + 1) - q0;
  const int k0 = __ldg(p.cu_k + s), lk = __ldg(p.cu_k + s + 1) - k0;
  const int key0 = jt * 128;
  if (key0 >= lk) return;  // the whole CTA leaves before any shared state exists

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sb = smem_u32(smem);
  // B_QF/B_QE, B_DF/B_DE: the Q and dO halves of the 2-stage ring, full / empty (Q is free once
  // dK(i) has read it, which is well before dV(i) frees dO, so Q(i+2) starts loading early);
  // B_STR: S^T(i) in TMEM; B_SF: dP^T(i) in TMEM (and dK(i-1) done); B_SE: S^T(i) read by the
  // elementwise warps (its columns may take S^T(i+1)); B_PF: P^T(i) in shared memory and dS^T(i)
  // in TMEM; B_PTE: dV(i) has read P^T(i).
  constexpr int B_KV = 0, B_QF = 1, B_QE = 3, B_DF = 5, B_DE = 7, B_SF = 9, B_SE = 10,
                B_PF = 11, B_PTE = 12, B_ACC = 13, B_DR = 14, B_STR = 15;
  constexpr int N_BARS = 16;
  static_assert(8 * N_BARS + 8 <= 256, "barrier area");
  const uint32_t bar0 = sb + L::SMEM_BAR;
#define TBAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::SMEM_BAR + 8 * N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned ecode = KID_BWD << 8;
  const uint64_t tmo = timeout_ns;

  const int shift = lk - lq;  // key position of query row i: i + shift
  const int it0 = CAUSAL ? max(0, key0 - shift) / 128 : 0;
  const int n_it = (lq + 127) / 128;
  const int nt = n_it - it0;
  const int n_iter = nt > 0 ? nt * p.R : 0;

  if (threadIdx.x == 0) {
    mbar_init(TBAR(B_KV), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(TBAR(B_QF + b), 1);
      mbar_init(TBAR(B_QE + b), 1);
      mbar_init(TBAR(B_DF + b), 1);
      mbar_init(TBAR(B_DE + b), 1);
    }
    mbar_init(TBAR(B_SF), 1);
    mbar_init(TBAR(B_SE), 4 * C::NWG);  // one elected arrival per elementwise warp
    mbar_init(TBAR(B_PF), 4 * C::NWG);
    mbar_init(TBAR(B_PTE), 1);
    mbar_init(TBAR(B_ACC), 1);
    mbar_init(TBAR(B_DR), 1);
    mbar_init(TBAR(B_STR), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::W_ISSUE) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D;

  if (warp == C::W_LOAD) {
    // ------------------------------------------------------------ TMA producer
    // lane 0: K, V, then the Q tiles; lane 1: the dO tiles (each on its own ring barriers)
    if (lane < 2) {
      const bool is_q = lane == 0;
      const int FB = is_q ? B_QF : B_DF, EB = is_q ? B_QE : B_DE;
      const CUtensorMap* tm = is_q ? &tm_q : &tm_do;
      const uint32_t off = is_q ? 0u : C::TILE_BYTES;
      uint32_t loaded = 0;
      bool ok = true;
      if (is_q) {
        mbar_arrive_expect_tx(TBAR(B_KV), 2 * C::TILE_BYTES);
#pragma unroll
        for (int a = 0; a < C::ATOMS; ++a) {
          tma_load_3d(sb + L::SMEM_K + a * C::ATOM_BYTES, &tm_k, TBAR(B_KV), a * 64, g,
                      k0 + key0);
          tma_load_3d(sb + L::SMEM_V + a * C::ATOM_BYTES, &tm_v, TBAR(B_KV), a * 64, g,
                      k0 + key0);
        }
      }
      for (int it = 0; it < n_iter && ok; ++it) {
        const int buf = it & 1;
        ok = mbar_wait(TBAR(EB + buf), ((it >> 1) & 1) ^ 1, abort_flag, tmo, ecode | 1);
        if (!ok) break;
        const int r = it / nt, i = it0 + it % nt;
        const int h = g * p.R + r;
        const int row = q0 + i * 128;
        const uint32_t dst = sb + L::SMEM_RING + buf * 2 * C::TILE_BYTES + off;
        mbar_arrive_expect_tx(TBAR(FB + buf), C::TILE_BYTES);
#pragma unroll
        for (int a = 0; a < C::ATOMS; ++a)
          tma_load_3d(dst + a * C::ATOM_BYTES, tm, TBAR(FB + buf), a * 64, h, row);
        ++loaded;
      }
      // Let every issued load land before shared memory goes away.
      volatile int never = 0;
      if (is_q) mbar_wait(TBAR(B_KV), 0, &never, tmo, ecode | 15);
      for (uint32_t it = (loaded > 2 ? loaded - 2 : 0); it < loaded; ++it)
        mbar_wait(TBAR(FB + (it & 1)), (it >> 1) & 1, &never, tmo, ecode | 15);
    }
  } else if (warp == C::W_ISSUE) {
    // ------------------------------------------------------------ tcgen05 issuer
    // Order: S^T(0), dP^T(0); then per iteration i: S^T(i+1) once the elementwise warps have
    // read S^T(i) (they exponentiate it while the tensor core runs the rest); once P^T(i) /
    // dS^T(i) are out: dK(i), dP^T(i+1) (the second phase of the next elementwise step waits
    // for these two GEMMs only), then dV(i) from the shared-memory P^T.
    if (lane == 0) {
      constexpr uint32_t ID_KK = umma_idesc_f16(BF16, 128, 128, false, false);  // both K-major
      constexpr uint32_t ID_PV = umma_idesc_f16(BF16, 128, D, false, true);     // B MN-major
      auto issue_st = [&](int it) {
        const uint32_t qs = sb + L::SMEM_RING + (it & 1) * 2 * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
          mma_ss(tmem + T_S, umma_desc_sw128(sb + L::SMEM_K + off, 16, 1024),
                 umma_desc_sw128(qs + off, 16, 1024), ID_KK, kk > 0 ? 1u : 0u);
        }
        mma_commit(TBAR(B_STR));
      };
      auto issue_dpt = [&](int it) {
        const uint32_t dos = sb + L::SMEM_RING + (it & 1) * 2 * C::TILE_BYTES + C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
          mma_ss(tmem + T_DP, umma_desc_sw128(sb + L::SMEM_V + off, 16, 1024),
                 umma_desc_sw128(dos + off, 16, 1024), ID_KK, kk > 0 ? 1u : 0u);
        }
        mma_commit(TBAR(B_SF));  // dP^T(i) (and everything issued before it)
      };
      bool ok = mbar_wait(TBAR(B_KV), 0, abort_flag, tmo, ecode | 2);
      tc_fence_after();
      if (ok && n_iter > 0) {
        ok = mbar_wait(TBAR(B_QF), 0, abort_flag, tmo, ecode | 3);
        tc_fence_after();
        if (ok) issue_st(0);
        if (ok) ok = mbar_wait(TBAR(B_DF), 0, abort_flag, tmo, ecode | 3);
        tc_fence_after();
        if (ok) issue_dpt(0);
      }
      for (int it = 0; it < n_iter && ok; ++it) {
        if (it + 1 < n_iter) {
          // ---- S^T(i+1) = K Q(i+1)^T into the columns S^T(i) was read from
          ok = mbar_wait_fast(TBAR(B_QF + ((it + 1) & 1)), ((it + 1) >> 1) & 1, abort_flag, tmo,
                         ecode | 3);
          if (ok) ok = mbar_wait_spin(TBAR(B_SE), it & 1, abort_flag, tmo, ecode | 7);
          if (!ok) break;
          tc_fence_after();
          issue_st(it + 1);
        }
        ok = mbar_wait_spin(TBAR(B_PF), it & 1, abort_flag, tmo, ecode | 4);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qs = sb + L::SMEM_RING + (it & 1) * 2 * C::TILE_BYTES;
        const uint32_t dos = qs + C::TILE_BYTES;
        // ---- dK += dS^T(i) Q(i)   (A: dS^T packed in TMEM); the last read of Q(i)
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16)
          mma_ts(tmem + T_DK, tmem + T_DP + C::packed_col(k16),
                 umma_desc_sw128(qs + k16 * 2048, C::ATOM_BYTES, 1024), ID_PV,
                 (it > 0 || k16 > 0) ? 1u : 0u);
        mma_commit(TBAR(B_QE + (it & 1)));
        // ---- dP^T(i+1) = V dO(i+1)^T over the dS^T(i) columns dK has just read
        if (it + 1 < n_iter) {
          ok = mbar_wait_fast(TBAR(B_DF + ((it + 1) & 1)), ((it + 1) >> 1) & 1, abort_flag, tmo,
                         ecode | 3);
          if (!ok) break;
          tc_fence_after();
          issue_dpt(it + 1);
        }
        // ---- dV += P^T(i) dO(i)   (A: P^T in shared memory, K-major)
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16) {
          const uint32_t off = (k16 >> 2) * C::ATOM_BYTES + (k16 & 3) * 32;
          mma_ss(tmem + T_DV, umma_desc_sw128(sb + L::SMEM_PT + off, 16, 1024),
                 umma_desc_sw128(dos + k16 * 2048, C::ATOM_BYTES, 1024), ID_PV,
                 (it > 0 || k16 > 0) ? 1u : 0u);
        }
        mma_commit(TBAR(B_PTE));
        mma_commit(TBAR(B_DE + (it & 1)));
      }
      mma_commit(TBAR(B_ACC));
      mma_commit(TBAR(B_DR));
      volatile int never = 0;
      mbar_wait(TBAR(B_DR), 0, &never, tmo, ecode | 14);
    }
  } else {
    // ------------------------------------------------------------ elementwise (thread = key)
    const int wg = threadIdx.x >> 7;                    // 32-row chunk of this warpgroup
    const int kl = threadIdx.x & 127;                   // key within the tile = TMEM lane
    const int key = key0 + kl;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    constexpr int BIAS = !ALIBI ? BIAS_NONE : (CAUSAL ? BIAS_LINEAR : BIAS_ABS);
    // this thread's row of P^T: the chunk's 64 bytes in atom wg / 2, 16-byte units
    // 4 (wg & 1) .. +3, 128-byte swizzle
    const uint32_t pt_row = sb + L::SMEM_PT + static_cast<uint32_t>(wg >> 1) * C::ATOM_BYTES +
                            static_cast<uint32_t>(kl) * 128u;
    const uint32_t sw = static_cast<uint32_t>(kl & 7);
    const uint64_t c1x2 = f2_pack(p.c1, p.c1);
    // Row terms of iteration it into L1 (two 128-byte lines each of na and nd for the chunk's
    // 32 rows), so the broadcast loads of the elementwise steps hit.
    auto prefetch_terms = [&](int it) {
      if (it >= n_iter || lane >= 4) return;
      const int r = it / nt, i = it0 + it % nt;
      const size_t w0 = static_cast<size_t>(g * p.R + r) * p.t_pad + q0 + i * 128 + wg * 32;
      prefetch_l1((lane < 2 ? p.na : p.nd) + w0 + (lane & 1) * 31);
    };
    prefetch_terms(0);
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      prefetch_terms(it + 1);
      const int r = it / nt, i = it0 + it % nt;
      const int h = g * p.R + r;
      const int rc0 = i * 128 + wg * 32;  // first row of this warpgroup's chunk
      float slope2 = 0.f;
      if constexpr (ALIBI) slope2 = __ldg(p.slopes + h) * LOG2E;
      // row terms of the chunk's 32 rows (pad rows past the last token keep these in bounds)
      const size_t wrow = static_cast<size_t>(h) * p.t_pad + q0 + rc0;
      const float* na_row = p.na + wrow;
      const float* nd_row = p.nd + wrow;
      // rows rc0 + e with e_lo <= e < e_hi see this key
      const int e_hi = key < lk ? min(32, lq - rc0) : 0;
      const int e_lo = CAUSAL ? key - shift - rc0 : 0;
      const bool full = __all_sync(0xffffffffu, e_lo <= 0 && e_hi >= 32);
      const float dd = static_cast<float>(rc0 + shift - key);
      const uint64_t kb2 = f2_pack(-slope2 * dd, -slope2 * dd);
      // ---- phase A: P from S^T(i)
      ok = mbar_wait(TBAR(B_STR), it & 1, abort_flag, tmo, ecode | 5);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float pr[32];
      {
        uint32_t sv[32];
        tmem_ld32(t_lane + T_S + wg * 32, sv);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(TBAR(B_SE));  // S^T(i) columns free for S^T(i+1)
        if (full)
          bwd_kv_p<false, BIAS>(sv, na_row, c1x2, kb2, slope2, dd, e_lo, e_hi, pr);
        else
          bwd_kv_p<true, BIAS>(sv, na_row, c1x2, kb2, slope2, dd, e_lo, e_hi, pr);
      }
      // ---- phase B: dS from dP^T(i), packed over the chunk's first 16 dP^T columns
      ok = mbar_wait(TBAR(B_SF), it & 1, abort_flag, tmo, ecode | 8);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t dv[16], pd[8];
        tmem_ld16(t_lane + T_DP + wg * 32, dv);
        tmem_wait_ld();
        bwd_kv_ds<BF16, 0>(pr, dv, nd_row, pd);
        tmem_st8(t_lane + T_DP + wg * 32, pd);
        tmem_ld16(t_lane + T_DP + wg * 32 + 16, dv);  // columns the store above did not touch
        tmem_wait_ld();
        bwd_kv_ds<BF16, 1>(pr, dv, nd_row, pd);
        tmem_st8(t_lane + T_DP + wg * 32 + 8, pd);
      }
      // P^T(i-1) has been read by dV(i-1) before P^T(i) goes over it.
      ok = mbar_wait(TBAR(B_PTE), (it - 1) & 1, abort_flag, tmo, ecode | 9);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        st_shared_v4(pt_row + ((static_cast<uint32_t>(4 * (wg & 1) + u) ^ sw) << 4),
                     bpack2<BF16>(pr[8 * u], pr[8 * u + 1]),
                     bpack2<BF16>(pr[8 * u + 2], pr[8 * u + 3]),
                     bpack2<BF16>(pr[8 * u + 4], pr[8 * u + 5]),
                     bpack2<BF16>(pr[8 * u + 6], pr[8 * u + 7]));
      // dS^T in TMEM and P^T in shared memory (generic proxy) reach the tensor core's reads.
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(TBAR(B_PF));
    }
    // ---- epilogue: dV, scale * dK for this thread's key
    if (ok) {
      ok = mbar_wait(TBAR(B_ACC), 0, abort_flag, tmo, ecode | 6);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      using OutT = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
      const bool any = n_iter > 0;
      const size_t o = (static_cast<size_t>(k0 + key) * p.hkv + g) * p.dh;
      // 32-byte stores (whole sectors, half the store instructions of 16-byte ones) while the
      // rows stay 32-byte aligned
      const bool kv_al32 =
          ((reinterpret_cast<uintptr_t>(p.dk) | reinterpret_cast<uintptr_t>(p.dv)) & 31) == 0 &&
          (p.dh & 15) == 0;
      // the first half of the groups writes dV, the second half scale * dK, each group its
      // share of the D columns
      constexpr int HALF = C::NWG / 2 > 0 ? C::NWG / 2 : 1;
      const bool is_v = C::NWG == 1 ? true : wg < HALF;
      const int part = C::NWG == 1 ? 0 : wg % HALF;
      const uint32_t src = is_v ? T_DV : T_DK;
      const float mul = is_v ? 1.f : p.scale;
      OutT* dst = reinterpret_cast<OutT*>(is_v ? p.dv : p.dk) + o;
      constexpr int CH = (D / 32) / HALF;  // 32-column chunks per group
#pragma unroll 1
      for (int c = part * CH; c < (part + 1) * CH; ++c) {
        uint32_t a[32];
        tmem_ld32(t_lane + src + c * 32, a);
        tmem_wait_ld();
        if (key < lk) {
          uint32_t pa[16];
#pragma unroll
          for (int u = 0; u < 16; ++u)
            pa[u] = any ? bpack2<BF16>(__uint_as_float(a[2 * u]) * mul,
                                       __uint_as_float(a[2 * u + 1]) * mul)
                        : 0u;
          if (kv_al32) {
#pragma unroll
            for (int i = 0; i < 2; ++i)
              if (c * 32 + i * 16 < p.dh) st_global_v8(dst + c * 32 + i * 16, &pa[8 * i]);
          } else {
            uint4* dp4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (c * 32 + u * 8 < p.dh)
                dp4[u] = make_uint4(pa[4 * u], pa[4 * u + 1], pa[4 * u + 2], pa[4 * u + 3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  asm volatile("bar.sync 0;" ::: "memory");
  if (warp == C::W_ISSUE) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
#undef TBAR
}

// -------------------------------------------------------------------------------------------
// dQ kernel layout: Q and dO of the current item; K in a 3-stage ring (its last use, dQ(j), comes
// a tile after S(j+2) would like to reuse the stage), V in a 2-stage ring (free after dP(j)).
template <int D>
struct BwdDqCfg {
  using T = BwdTcCfg<D>;
  static constexpr uint32_t SMEM_Q = 0, SMEM_DO = T::TILE_BYTES;
  static constexpr uint32_t SMEM_K = 2 * T::TILE_BYTES;   // 3 stages
  static constexpr uint32_t SMEM_V = 5 * T::TILE_BYTES;   // 2 stages
  static constexpr uint32_t SMEM_BAR = 7 * T::TILE_BYTES;
  static constexpr uint32_t SMEM_TOTAL = SMEM_BAR + 256 + 1024;
  static_assert(SMEM_TOTAL <= 232448, "shared memory per CTA");
};

// Grid: x = query tile * (hq / mq) + group of mq query heads (causal: the last tiles, which see
// the most keys, first), y = segment in the pre kernel's order (heaviest first).
template <int D, bool BF16, bool CAUSAL, bool ALIBI>
__global__ void __launch_bounds__(BwdTcCfg<D>::THREADS, 1)
    mea_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const BwdParams p,
                         unsigned long long timeout_ns) {
  using C = BwdTcCfg<D>;
  using L = BwdDqCfg<D>;
  constexpr float LOG2E = 1.4426950408889634f;
  const int n_grp = p.hq / p.mq, bx = static_cast<int>(blockIdx.x);
  const int n_tiles = static_cast<int>(gridDim.x) / n_grp, tl = bx / n_grp;
  const int itile = CAUSAL ? n_tiles - 1 - tl : tl;
  const int s = p.order ? p.order[blockIdx.y] : blockIdx.y;
  const int h0 = (bx - tl * n_grp) * p.mq, n_items = p.mq;
  const int q0 = __ldg(p.cu_q + s), lq = __ldg(p.cu_q + s + 1) - q0;
  const int k0 = __ldg(p.cu_k + s), lk = __ldg(p.cu_k + s + 1) - k0;
  const int row0 = itile * 128;
  if (row0 >= lq) return;  // the whole CTA leaves before any shared state exists

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sb = smem_u32(smem);
  // Per tile (gt counts tiles over the CTA's items): B_KF/B_KE the K ring (3), B_VF/B_VE the V
  // ring (2), B_SF S(gt) and dP(gt) in TMEM, B_PF dS(gt) packed by the elementwise warps. Per item
  // (m): B_QF/B_QE Q and dO loaded / no longer read, B_ACC dQ complete, B_DQE dQ read out of TMEM
  // by the elementwise warps (the next item may accumulate over it).
  constexpr int B_QF = 0, B_KF = 1, B_KE = 4, B_VF = 7, B_VE = 9, B_SF = 11, B_PF = 12,
                B_ACC = 13, B_DR = 14, B_QE = 15, B_DQE = 16;
  constexpr int N_BARS = 17;
  static_assert(8 * N_BARS + 8 <= 256, "barrier area");
  const uint32_t bar0 = sb + L::SMEM_BAR;
#define TBAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::SMEM_BAR + 8 * N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned ecode = (KID_BWD << 8) | 0x80;
  const uint64_t tmo = timeout_ns;

  // Every item of the CTA covers the same rows, hence the same key tiles.
  const int shift = lk - lq;
  const int nrows = min(128, lq - row0);
  int n_jt = (lk + 127) / 128;
  if (CAUSAL) {
    const int kmax = min(lk - 1, row0 + nrows - 1 + shift);
    n_jt = kmax >= 0 ? kmax / 128 + 1 : 0;
  }

  if (threadIdx.x == 0) {
    mbar_init(TBAR(B_QF), 1);
    mbar_init(TBAR(B_QE), 1);
    for (int b = 0; b < 3; ++b) {
      mbar_init(TBAR(B_KF + b), 1);
      mbar_init(TBAR(B_KE + b), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(TBAR(B_VF + b), 1);
      mbar_init(TBAR(B_VE + b), 1);
    }
    mbar_init(TBAR(B_SF), 1);
    mbar_init(TBAR(B_PF), 4 * C::NWG);   // one elected arrival per elementwise warp
    mbar_init(TBAR(B_ACC), 1);
    mbar_init(TBAR(B_DR), 1);
    mbar_init(TBAR(B_DQE), 4 * C::NWG);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::W_ISSUE) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM: S(gt) in buffer gt mod 2, then dP and the dQ accumulator.
  const uint32_t T_S0 = 0, T_DP = 256, T_DQ = 384;

  if (warp == C::W_LOAD) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      uint32_t gk = 0, gv = 0;  // K / V tiles loaded over the CTA's items
      int nq = 0;               // items whose Q / dO were issued
      for (int m = 0; m < n_items && ok; ++m) {
        const int h = h0 + m, g = h / p.R;
        // Q and dO of item m, once the previous item no longer reads them
        ok = mbar_wait(TBAR(B_QE), (m & 1) ^ 1, abort_flag, tmo, ecode | 1);
        if (!ok) break;
        if (n_jt > 0) {
          mbar_arrive_expect_tx(TBAR(B_QF), 2 * C::TILE_BYTES);
#pragma unroll
          for (int a = 0; a < C::ATOMS; ++a) {
            tma_load_3d(sb + L::SMEM_Q + a * C::ATOM_BYTES, &tm_q, TBAR(B_QF), a * 64, h,
                        q0 + row0);
            tma_load_3d(sb + L::SMEM_DO + a * C::ATOM_BYTES, &tm_do, TBAR(B_QF), a * 64, h,
                        q0 + row0);
          }
        } else {
          mbar_arrive(TBAR(B_QF));
        }
        nq = m + 1;
        for (int jt = 0; jt < n_jt && ok; ++jt) {
          const uint32_t kb = gk % 3, vb = gv & 1;
          ok = mbar_wait(TBAR(B_KE + kb), ((gk / 3) & 1) ^ 1, abort_flag, tmo, ecode | 1);
          if (!ok) break;
          mbar_arrive_expect_tx(TBAR(B_KF + kb), C::TILE_BYTES);
#pragma unroll
          for (int a = 0; a < C::ATOMS; ++a)
            tma_load_3d(sb + L::SMEM_K + kb * C::TILE_BYTES + a * C::ATOM_BYTES, &tm_k,
                        TBAR(B_KF + kb), a * 64, g, k0 + jt * 128);
          ++gk;
          ok = mbar_wait(TBAR(B_VE + vb), ((gv >> 1) & 1) ^ 1, abort_flag, tmo, ecode | 1);
          if (!ok) break;
          mbar_arrive_expect_tx(TBAR(B_VF + vb), C::TILE_BYTES);
#pragma unroll
          for (int a = 0; a < C::ATOMS; ++a)
            tma_load_3d(sb + L::SMEM_V + vb * C::TILE_BYTES + a * C::ATOM_BYTES, &tm_v,
                        TBAR(B_VF + vb), a * 64, g, k0 + jt * 128);
          ++gv;
        }
      }
      // Let every issued load land before shared memory goes away.
      volatile int never = 0;
      if (nq > 0) mbar_wait(TBAR(B_QF), (nq - 1) & 1, &never, tmo, ecode | 15);
      for (uint32_t x = (gk > 3 ? gk - 3 : 0); x < gk; ++x)
        mbar_wait(TBAR(B_KF + x % 3), (x / 3) & 1, &never, tmo, ecode | 15);
      for (uint32_t x = (gv > 2 ? gv - 2 : 0); x < gv; ++x)
        mbar_wait(TBAR(B_VF + (x & 1)), (x >> 1) & 1, &never, tmo, ecode | 15);
    }
  } else if (warp == C::W_ISSUE) {
    // ------------------------------------------------------------ tcgen05 issuer
    // Per item: S(0), dP(0), S(1); then per tile j, once dS(j) is packed: dP(j+1) (the next
    // elementwise step waits for that one GEMM only, S(j+1) being already there), dQ(j) (the
    // item's first one waits until the previous item's dQ has been read out of TMEM), then
    // S(j+2) into the buffer dQ(j) has just read. Once the item's last dP is issued, its Q / dO
    // go back to the producer, which loads the next item's while this one finishes.
    if (lane == 0) {
      constexpr uint32_t ID_KK = umma_idesc_f16(BF16, 128, 128, false, false);
      constexpr uint32_t ID_PV = umma_idesc_f16(BF16, 128, D, false, true);
      auto issue_s = [&](uint32_t gt) -> bool {
        const uint32_t kb = gt % 3;
        if (!mbar_wait_fast(TBAR(B_KF + kb), (gt / 3) & 1, abort_flag, tmo, ecode | 3))
          return false;
        tc_fence_after();
        const uint32_t ks = sb + L::SMEM_K + kb * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
          mma_ss(tmem + T_S0 + (gt & 1) * 128, umma_desc_sw128(sb + L::SMEM_Q + off, 16, 1024),
                 umma_desc_sw128(ks + off, 16, 1024), ID_KK, kk > 0 ? 1u : 0u);
        }
        return true;
      };
      auto issue_dp = [&](uint32_t gt) -> bool {
        const uint32_t vb = gt & 1;
        if (!mbar_wait_fast(TBAR(B_VF + vb), (gt >> 1) & 1, abort_flag, tmo, ecode | 3))
          return false;
        tc_fence_after();
        const uint32_t vs = sb + L::SMEM_V + vb * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
          mma_ss(tmem + T_DP, umma_desc_sw128(sb + L::SMEM_DO + off, 16, 1024),
                 umma_desc_sw128(vs + off, 16, 1024), ID_KK, kk > 0 ? 1u : 0u);
        }
        mma_commit(TBAR(B_VE + vb));
        mma_commit(TBAR(B_SF));  // S(gt) (issued earlier) and dP(gt)
        return true;
      };
      bool ok = true;
      const uint32_t n = static_cast<uint32_t>(n_jt);
      for (int m = 0; m < n_items && ok; ++m) {
        const uint32_t g = static_cast<uint32_t>(m) * n;  // tiles of the previous items
        ok = mbar_wait(TBAR(B_QF), m & 1, abort_flag, tmo, ecode | 2);
        if (!ok) break;
        tc_fence_after();
        if (n > 0) {
          ok = issue_s(g) && issue_dp(g);
          if (ok && n == 1) mma_commit(TBAR(B_QE));
          if (ok && n > 1) ok = issue_s(g + 1);
        } else {
          // No tiles: B_ACC(m) still waits for the read-out of item m-1, so that the per-item
          // barriers never run two phases ahead of the elementwise warps.
          mma_commit(TBAR(B_QE));
          ok = mbar_wait_spin(TBAR(B_DQE), (m & 1) ^ 1, abort_flag, tmo, ecode | 7);
        }
        for (uint32_t jt = 0; jt < n && ok; ++jt) {
          const uint32_t gt = g + jt;
          ok = mbar_wait_spin(TBAR(B_PF), gt & 1, abort_flag, tmo, ecode | 4);
          if (!ok) break;
          tc_fence_after();
          if (jt + 1 < n) {
            if (!(ok = issue_dp(gt + 1))) break;
            if (jt + 2 == n) mma_commit(TBAR(B_QE));  // the item's last read of Q / dO
          }
          if (jt == 0) {
            // the previous item's dQ has been read out of TMEM
            ok = mbar_wait_spin(TBAR(B_DQE), (m & 1) ^ 1, abort_flag, tmo, ecode | 7);
            if (!ok) break;
            tc_fence_after();
          }
          // ---- dQ += dS(j) K(j)
          const uint32_t ks = sb + L::SMEM_K + (gt % 3) * C::TILE_BYTES;
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            mma_ts(tmem + T_DQ, tmem + T_S0 + (gt & 1) * 128 + C::packed_col(k16),
                   umma_desc_sw128(ks + k16 * 2048, C::ATOM_BYTES, 1024), ID_PV,
                   (jt > 0 || k16 > 0) ? 1u : 0u);
          mma_commit(TBAR(B_KE + gt % 3));
          if (jt + 2 < n && !(ok = issue_s(gt + 2))) break;
        }
        if (ok) mma_commit(TBAR(B_ACC));
      }
      mma_commit(TBAR(B_DR));
      volatile int never = 0;
      mbar_wait(TBAR(B_DR), 0, &never, tmo, ecode | 14);
    }
  } else {
    // ------------------------------------------------------------ elementwise (thread = row)
    const int wg = threadIdx.x >> 7;                    // column quarter of this warpgroup
    const int rl = threadIdx.x & 127;
    const int row = row0 + rl;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    constexpr int BIAS = !ALIBI ? BIAS_NONE : (CAUSAL ? BIAS_LINEAR : BIAS_ABS);
    const uint64_t c1x2 = f2_pack(p.c1, p.c1);
    using OutT = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    bool ok = true;
    for (int m = 0; m < n_items && ok; ++m) {
      const int h = h0 + m;
      const uint32_t g = static_cast<uint32_t>(m * n_jt);  // tiles of the previous items
      const size_t li = static_cast<size_t>(h) * p.total_q + q0 + row;
      const float lse2 = row < lq ? __ldg(p.lse + li) * LOG2E : 0.f;
      const float dl = row < lq ? -p.nd[static_cast<size_t>(h) * p.t_pad + q0 + row] : 0.f;
      float slope2 = 0.f;
      if constexpr (ALIBI) slope2 = __ldg(p.slopes + h) * LOG2E;
      const uint64_t nd2 = f2_pack(-dl, -dl);
      for (int jt = 0; jt < n_jt && ok; ++jt) {
        const uint32_t gt = g + static_cast<uint32_t>(jt);
        ok = mbar_wait(TBAR(B_SF), gt & 1, abort_flag, tmo, ecode | 5);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t t_s = T_S0 + (gt & 1) * 128;
#pragma unroll 1
        for (int cc = 0; cc < C::CPW; ++cc) {
          const int c = C::CPW * wg + cc;
          uint32_t sv[32], dv[32];
          tmem_ld32(t_lane + t_s + c * 32, sv);
          tmem_ld32(t_lane + T_DP + c * 32, dv);
          // keys kc0 + e with e < e_hi are seen by this row
          const int kc0 = jt * 128 + c * 32;
          const int dk = row + shift - kc0;
          int e_hi = row < lq ? min(32, lk - kc0) : 0;
          if (CAUSAL) e_hi = min(e_hi, dk + 1);
          const bool full = __all_sync(0xffffffffu, e_hi >= 32);
          float b = -lse2;
          if constexpr (BIAS == BIAS_LINEAR) b = fmaf(-slope2, static_cast<float>(dk), b);
          tmem_wait_ld();
          const uint32_t t_d = t_lane + t_s + 32 * C::CPW * wg + cc * 16;
          if (full)
            bwd_q_chunk<BF16, false, BIAS>(sv, dv, c1x2, b, slope2, static_cast<float>(dk), nd2,
                                           e_hi, t_d);
          else
            bwd_q_chunk<BF16, true, BIAS>(sv, dv, c1x2, b, slope2, static_cast<float>(dk), nd2,
                                          e_hi, t_d);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(TBAR(B_PF));
      }
      if (!ok) break;
      // ---- dQ out of TMEM, scaled and packed; group w holds chunk w of the D columns (groups
      // past D/32 hold none)
      ok = mbar_wait(TBAR(B_ACC), m & 1, abort_flag, tmo, ecode | 6);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const bool any = n_jt > 0;
      // 32-byte stores while the rows stay 32-byte aligned (as for dK/dV)
      const bool dq_al32 = (reinterpret_cast<uintptr_t>(p.dq) & 31) == 0 && (p.dh & 15) == 0;
      if (wg < D / 32) {
        uint32_t a[32];
        tmem_ld32(t_lane + T_DQ + wg * 32, a);
        tmem_wait_ld();
        if (row < lq) {
          uint32_t pa[16];
#pragma unroll
          for (int u = 0; u < 16; ++u)
            pa[u] = any ? bpack2<BF16>(__uint_as_float(a[2 * u]) * p.scale,
                                       __uint_as_float(a[2 * u + 1]) * p.scale)
                        : 0u;
          const size_t o = (static_cast<size_t>(q0 + row) * p.hq + h) * p.dh;
          OutT* dqrow = reinterpret_cast<OutT*>(p.dq) + o + wg * 32;
          if (dq_al32) {
#pragma unroll
            for (int i = 0; i < 2; ++i)
              if (wg * 32 + i * 16 < p.dh) st_global_v8(dqrow + i * 16, &pa[8 * i]);
          } else {
            uint4* dqp = reinterpret_cast<uint4*>(dqrow);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (wg * 32 + u * 8 < p.dh)
                dqp[u] = make_uint4(pa[4 * u], pa[4 * u + 1], pa[4 * u + 2], pa[4 * u + 3]);
          }
        }
      }
      // dQ has been read out of TMEM: the next item may accumulate over it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(TBAR(B_DQE));
    }
  }
  tc_fence_before();
  asm volatile("bar.sync 0;" ::: "memory");
  if (warp == C::W_ISSUE) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
#undef TBAR
}

}  // namespace mea
