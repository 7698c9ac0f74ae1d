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
//   P^T, dS^T                        (elementwise warpgroup: thread = key = TMEM lane), written
//                                    bf16/f16-packed over the first 64 columns of S^T / dP^T
//   dV += P^T dO, dK += dS^T Q       (tcgen05, A from TMEM, B = the [rows][D] tiles MN-major)
// TMEM: S^T [0,128), dP^T [128,256), dV [256,256+D), dK [256+D,256+2D). dK and dV accumulate
// over the whole GQA group; they are written once.
//
// mea_bwd_dq_tc_kernel: one CTA per (128-row query tile, segment, query head), over the key
// tiles the rows see: S = Q K^T, dP = dO V^T, dS (thread = row), dQ += dS K.
// TMEM: S [0,128), dP [128,256), dQ [256,256+D).
//
// Roles (NWG*128 + 64 threads): NWG elementwise warpgroups (thread = TMEM lane; group w handles
// the 32-column chunks [128w/NWG, 128(w+1)/NWG) of the S/dP tiles and writes its packed P / dS
// over the first half of its own columns, so the groups never touch each other's columns), warp
// 4*NWG the tcgen05 issuer (owns TMEM), warp 4*NWG+1 the TMA producer. Every wait is bounded; no
// named barriers in the role loops.
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
  static constexpr uint32_t SMEM_A = 0;                  // K (dkdv) / Q (dq), loaded once
  static constexpr uint32_t SMEM_B = TILE_BYTES;         // V (dkdv) / dO (dq), loaded once
  static constexpr uint32_t SMEM_RING = 2 * TILE_BYTES;  // 2 stages x 2 tiles
  static constexpr uint32_t SMEM_BAR = SMEM_RING + 4 * TILE_BYTES;
  static constexpr uint32_t SMEM_TOTAL = SMEM_BAR + 256 + 1024;
  static_assert(SMEM_TOTAL <= 232448, "shared memory per CTA");
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

// -------------------------------------------------------------------------------------------
template <int D, bool BF16, bool CAUSAL, bool ALIBI>
__global__ void __launch_bounds__(BwdTcCfg<D>::THREADS, 1)
    mea_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_do,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const BwdParams p,
                           unsigned long long timeout_ns) {
  using C = BwdTcCfg<D>;
  constexpr float LOG2E = 1.4426950408889634f;
  const int jt = blockIdx.x, s = blockIdx.y, g = blockIdx.z;
  const int q0 = __ldg(p.cu_q + s), lq = __ldg(p.cu_q + s + 1) - q0;
  const int k0 = __ldg(p.cu_k + s), lk = __ldg(p.cu_k + s + 1) - k0;
  const int key0 = jt * 128;
  if (key0 >= lk) return;  // the whole CTA leaves before any shared state exists

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sb = smem_u32(smem);
  constexpr int B_KV = 0, B_QF = 1, B_QE = 3, B_SF = 5, B_PF = 6, B_ACC = 7, B_DR = 8;
  constexpr int N_BARS = 9;
  const uint32_t bar0 = sb + C::SMEM_BAR;
#define TBAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_BAR + 8 * N_BARS);
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
    }
    mbar_init(TBAR(B_SF), 1);
    mbar_init(TBAR(B_PF), 4 * C::NWG);  // one elected arrival per elementwise warp
    mbar_init(TBAR(B_ACC), 1);
    mbar_init(TBAR(B_DR), 1);
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
    if (lane == 0) {
      uint32_t loaded = 0;
      bool ok = true;
      mbar_arrive_expect_tx(TBAR(B_KV), 2 * C::TILE_BYTES);
#pragma unroll
      for (int a = 0; a < C::ATOMS; ++a) {
        tma_load_3d(sb + C::SMEM_A + a * C::ATOM_BYTES, &tm_k, TBAR(B_KV), a * 64, g, k0 + key0);
        tma_load_3d(sb + C::SMEM_B + a * C::ATOM_BYTES, &tm_v, TBAR(B_KV), a * 64, g, k0 + key0);
      }
      for (int it = 0; it < n_iter && ok; ++it) {
        const int buf = it & 1;
        ok = mbar_wait(TBAR(B_QE + buf), ((it >> 1) & 1) ^ 1, abort_flag, tmo, ecode | 1);
        if (!ok) break;
        const int r = it / nt, i = it0 + it % nt;
        const int h = g * p.R + r;
        const int row = q0 + i * 128;
        const uint32_t qs = sb + C::SMEM_RING + buf * 2 * C::TILE_BYTES;
        mbar_arrive_expect_tx(TBAR(B_QF + buf), 2 * C::TILE_BYTES);
#pragma unroll
        for (int a = 0; a < C::ATOMS; ++a) {
          tma_load_3d(qs + a * C::ATOM_BYTES, &tm_q, TBAR(B_QF + buf), a * 64, h, row);
          tma_load_3d(qs + C::TILE_BYTES + a * C::ATOM_BYTES, &tm_do, TBAR(B_QF + buf), a * 64, h,
                      row);
        }
        ++loaded;
      }
      // Let every issued load land before shared memory goes away.
      volatile int never = 0;
      mbar_wait(TBAR(B_KV), 0, &never, tmo, ecode | 15);
      for (uint32_t it = (loaded > 2 ? loaded - 2 : 0); it < loaded; ++it)
        mbar_wait(TBAR(B_QF + (it & 1)), (it >> 1) & 1, &never, tmo, ecode | 15);
    }
  } else if (warp == C::W_ISSUE) {
    // ------------------------------------------------------------ tcgen05 issuer
    if (lane == 0) {
      constexpr uint32_t ID_KK = umma_idesc_f16(BF16, 128, 128, false, false);  // both K-major
      constexpr uint32_t ID_PV = umma_idesc_f16(BF16, 128, D, false, true);     // B MN-major
      bool ok = mbar_wait(TBAR(B_KV), 0, abort_flag, tmo, ecode | 2);
      tc_fence_after();
      for (int it = 0; it <= n_iter && ok; ++it) {
        const int buf = it & 1;
        if (it < n_iter) {
          ok = mbar_wait(TBAR(B_QF + buf), (it >> 1) & 1, abort_flag, tmo, ecode | 3);
          if (!ok) break;
          tc_fence_after();
        }
        if (it > 0) {
          // ---- dV += P^T dO, dK += dS^T Q for iteration it-1
          ok = mbar_wait_spin(TBAR(B_PF), (it - 1) & 1, abort_flag, tmo, ecode | 4);
          if (!ok) break;
          tc_fence_after();
          const uint32_t qs = sb + C::SMEM_RING + ((it - 1) & 1) * 2 * C::TILE_BYTES;
          const uint32_t dos = qs + C::TILE_BYTES;
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            mma_ts(tmem + T_DV, tmem + T_S + C::packed_col(k16),
                   umma_desc_sw128(dos + k16 * 2048, C::ATOM_BYTES, 1024), ID_PV,
                   (it - 1 > 0 || k16 > 0) ? 1u : 0u);
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            mma_ts(tmem + T_DK, tmem + T_DP + C::packed_col(k16),
                   umma_desc_sw128(qs + k16 * 2048, C::ATOM_BYTES, 1024), ID_PV,
                   (it - 1 > 0 || k16 > 0) ? 1u : 0u);
          mma_commit(TBAR(B_QE + ((it - 1) & 1)));
        }
        if (it < n_iter) {
          // ---- S^T = K Q^T, dP^T = V dO^T
          const uint32_t qs = sb + C::SMEM_RING + buf * 2 * C::TILE_BYTES;
          const uint32_t dos = qs + C::TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
            mma_ss(tmem + T_S, umma_desc_sw128(sb + C::SMEM_A + off, 16, 1024),
                   umma_desc_sw128(qs + off, 16, 1024), ID_KK, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
            mma_ss(tmem + T_DP, umma_desc_sw128(sb + C::SMEM_B + off, 16, 1024),
                   umma_desc_sw128(dos + off, 16, 1024), ID_KK, kk > 0 ? 1u : 0u);
          }
          mma_commit(TBAR(B_SF));
        }
      }
      mma_commit(TBAR(B_ACC));
      mma_commit(TBAR(B_DR));
      volatile int never = 0;
      mbar_wait(TBAR(B_DR), 0, &never, tmo, ecode | 14);
    }
  } else {
    // ------------------------------------------------------------ elementwise (thread = key)
    const int wg = threadIdx.x >> 7;                    // column half of this warpgroup
    const int kl = threadIdx.x & 127;                   // key within the tile = TMEM lane
    const int key = key0 + kl;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      ok = mbar_wait(TBAR(B_SF), it & 1, abort_flag, tmo, ecode | 5);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int r = it / nt, i = it0 + it % nt;
      const int h = g * p.R + r;
      const int row0 = i * 128;
      float slope2 = 0.f;
      if constexpr (ALIBI) slope2 = __ldg(p.slopes + h) * LOG2E;
#pragma unroll 1
      for (int cc = 0; cc < C::CPW; ++cc) {
        const int c = C::CPW * wg + cc;       // 32-column chunk of the tile
        uint32_t sv[32], dv[32];
        tmem_ld32(t_lane + T_S + c * 32, sv);
        tmem_ld32(t_lane + T_DP + c * 32, dv);
        const int rr = row0 + c * 32 + lane;  // this lane fetches the row values of column rr
        const size_t li = static_cast<size_t>(h) * p.total_q + q0 + rr;
        const float lse_l = rr < lq ? __ldg(p.lse + li) * LOG2E : 0.f;
        const float dl_l = rr < lq ? p.delta[li] : 0.f;
        tmem_wait_ld();
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float pe[2], de[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int row = row0 + c * 32 + e + u;
            const float lse_e = __shfl_sync(0xffffffffu, lse_l, e + u);
            const float dl_e = __shfl_sync(0xffffffffu, dl_l, e + u);
            const bool valid = row < lq && key < lk && (!CAUSAL || key <= row + shift);
            float z = __uint_as_float(sv[e + u]) * p.c1 - lse_e;
            if constexpr (ALIBI) z -= slope2 * fabsf(static_cast<float>(row + shift - key));
            const float pv = valid ? ex2_approx(z) : 0.f;
            pe[u] = pv;
            de[u] = pv * (__uint_as_float(dv[e + u]) - dl_e);
          }
          pp[e >> 1] = bpack2<BF16>(pe[0], pe[1]);
          pd[e >> 1] = bpack2<BF16>(de[0], de[1]);
        }
        tmem_st16(t_lane + T_S + 32 * C::CPW * wg + cc * 16, pp);
        tmem_st16(t_lane + T_DP + 32 * C::CPW * wg + cc * 16, pd);
      }
      tmem_wait_st();
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
          uint4* dp4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (c * 32 + u * 8 < p.dh)
              dp4[u] = make_uint4(pa[4 * u], pa[4 * u + 1], pa[4 * u + 2], pa[4 * u + 3]);
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
template <int D, bool BF16, bool CAUSAL, bool ALIBI>
__global__ void __launch_bounds__(BwdTcCfg<D>::THREADS, 1)
    mea_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const BwdParams p,
                         unsigned long long timeout_ns) {
  using C = BwdTcCfg<D>;
  constexpr float LOG2E = 1.4426950408889634f;
  // Causal: the last query tiles see the most keys; start them first.
  const int itile = CAUSAL ? static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x)
                           : static_cast<int>(blockIdx.x);
  const int s = blockIdx.y, h = blockIdx.z, g = h / p.R;
  const int q0 = __ldg(p.cu_q + s), lq = __ldg(p.cu_q + s + 1) - q0;
  const int k0 = __ldg(p.cu_k + s), lk = __ldg(p.cu_k + s + 1) - k0;
  const int row0 = itile * 128;
  if (row0 >= lq) return;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sb = smem_u32(smem);
  constexpr int B_QD = 0, B_KF = 1, B_KE = 3, B_SF = 5, B_PF = 6, B_ACC = 7, B_DR = 8;
  constexpr int N_BARS = 9;
  const uint32_t bar0 = sb + C::SMEM_BAR;
#define TBAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_BAR + 8 * N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned ecode = (KID_BWD << 8) | 0x80;
  const uint64_t tmo = timeout_ns;

  const int shift = lk - lq;
  const int nrows = min(128, lq - row0);
  int n_jt = (lk + 127) / 128;
  if (CAUSAL) {
    const int kmax = min(lk - 1, row0 + nrows - 1 + shift);
    n_jt = kmax >= 0 ? kmax / 128 + 1 : 0;
  }

  if (threadIdx.x == 0) {
    mbar_init(TBAR(B_QD), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(TBAR(B_KF + b), 1);
      mbar_init(TBAR(B_KE + b), 1);
    }
    mbar_init(TBAR(B_SF), 1);
    mbar_init(TBAR(B_PF), 4 * C::NWG);  // one elected arrival per elementwise warp
    mbar_init(TBAR(B_ACC), 1);
    mbar_init(TBAR(B_DR), 1);
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
  const uint32_t T_S = 0, T_DP = 128, T_DQ = 256;

  if (warp == C::W_LOAD) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t loaded = 0;
      bool ok = true;
      mbar_arrive_expect_tx(TBAR(B_QD), 2 * C::TILE_BYTES);
#pragma unroll
      for (int a = 0; a < C::ATOMS; ++a) {
        tma_load_3d(sb + C::SMEM_A + a * C::ATOM_BYTES, &tm_q, TBAR(B_QD), a * 64, h, q0 + row0);
        tma_load_3d(sb + C::SMEM_B + a * C::ATOM_BYTES, &tm_do, TBAR(B_QD), a * 64, h, q0 + row0);
      }
      for (int jt = 0; jt < n_jt && ok; ++jt) {
        const int buf = jt & 1;
        ok = mbar_wait(TBAR(B_KE + buf), ((jt >> 1) & 1) ^ 1, abort_flag, tmo, ecode | 1);
        if (!ok) break;
        const uint32_t ks = sb + C::SMEM_RING + buf * 2 * C::TILE_BYTES;
        mbar_arrive_expect_tx(TBAR(B_KF + buf), 2 * C::TILE_BYTES);
#pragma unroll
        for (int a = 0; a < C::ATOMS; ++a) {
          tma_load_3d(ks + a * C::ATOM_BYTES, &tm_k, TBAR(B_KF + buf), a * 64, g, k0 + jt * 128);
          tma_load_3d(ks + C::TILE_BYTES + a * C::ATOM_BYTES, &tm_v, TBAR(B_KF + buf), a * 64, g,
                      k0 + jt * 128);
        }
        ++loaded;
      }
      volatile int never = 0;
      mbar_wait(TBAR(B_QD), 0, &never, tmo, ecode | 15);
      for (uint32_t jt = (loaded > 2 ? loaded - 2 : 0); jt < loaded; ++jt)
        mbar_wait(TBAR(B_KF + (jt & 1)), (jt >> 1) & 1, &never, tmo, ecode | 15);
    }
  } else if (warp == C::W_ISSUE) {
    // ------------------------------------------------------------ tcgen05 issuer
    if (lane == 0) {
      constexpr uint32_t ID_KK = umma_idesc_f16(BF16, 128, 128, false, false);
      constexpr uint32_t ID_PV = umma_idesc_f16(BF16, 128, D, false, true);
      bool ok = mbar_wait(TBAR(B_QD), 0, abort_flag, tmo, ecode | 2);
      tc_fence_after();
      for (int jt = 0; jt <= n_jt && ok; ++jt) {
        const int buf = jt & 1;
        if (jt < n_jt) {
          ok = mbar_wait(TBAR(B_KF + buf), (jt >> 1) & 1, abort_flag, tmo, ecode | 3);
          if (!ok) break;
          tc_fence_after();
        }
        if (jt > 0) {
          // ---- dQ += dS K for key tile jt-1
          ok = mbar_wait_spin(TBAR(B_PF), (jt - 1) & 1, abort_flag, tmo, ecode | 4);
          if (!ok) break;
          tc_fence_after();
          const uint32_t ks = sb + C::SMEM_RING + ((jt - 1) & 1) * 2 * C::TILE_BYTES;
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            mma_ts(tmem + T_DQ, tmem + T_S + C::packed_col(k16),
                   umma_desc_sw128(ks + k16 * 2048, C::ATOM_BYTES, 1024), ID_PV,
                   (jt - 1 > 0 || k16 > 0) ? 1u : 0u);
          mma_commit(TBAR(B_KE + ((jt - 1) & 1)));
        }
        if (jt < n_jt) {
          // ---- S = Q K^T, dP = dO V^T
          const uint32_t ks = sb + C::SMEM_RING + buf * 2 * C::TILE_BYTES;
          const uint32_t vs = ks + C::TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
            mma_ss(tmem + T_S, umma_desc_sw128(sb + C::SMEM_A + off, 16, 1024),
                   umma_desc_sw128(ks + off, 16, 1024), ID_KK, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
            mma_ss(tmem + T_DP, umma_desc_sw128(sb + C::SMEM_B + off, 16, 1024),
                   umma_desc_sw128(vs + off, 16, 1024), ID_KK, kk > 0 ? 1u : 0u);
          }
          mma_commit(TBAR(B_SF));
        }
      }
      mma_commit(TBAR(B_ACC));
      mma_commit(TBAR(B_DR));
      volatile int never = 0;
      mbar_wait(TBAR(B_DR), 0, &never, tmo, ecode | 14);
    }
  } else {
    // ------------------------------------------------------------ elementwise (thread = row)
    const int wg = threadIdx.x >> 7;                    // column half of this warpgroup
    const int rl = threadIdx.x & 127;
    const int row = row0 + rl;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const size_t li = static_cast<size_t>(h) * p.total_q + q0 + row;
    const float lse2 = row < lq ? __ldg(p.lse + li) * LOG2E : 0.f;
    const float dl = row < lq ? p.delta[li] : 0.f;
    float slope2 = 0.f;
    if constexpr (ALIBI) slope2 = __ldg(p.slopes + h) * LOG2E;
    bool ok = true;
    for (int jt = 0; jt < n_jt && ok; ++jt) {
      ok = mbar_wait(TBAR(B_SF), jt & 1, abort_flag, tmo, ecode | 5);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < C::CPW; ++cc) {
        const int c = C::CPW * wg + cc;
        uint32_t sv[32], dv[32];
        tmem_ld32(t_lane + T_S + c * 32, sv);
        tmem_ld32(t_lane + T_DP + c * 32, dv);
        tmem_wait_ld();
        uint32_t pd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float de[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int key = jt * 128 + c * 32 + e + u;
            const bool valid = row < lq && key < lk && (!CAUSAL || key <= row + shift);
            float z = __uint_as_float(sv[e + u]) * p.c1 - lse2;
            if constexpr (ALIBI) z -= slope2 * fabsf(static_cast<float>(row + shift - key));
            const float pv = valid ? ex2_approx(z) : 0.f;
            de[u] = pv * (__uint_as_float(dv[e + u]) - dl);
          }
          pd[e >> 1] = bpack2<BF16>(de[0], de[1]);
        }
        tmem_st16(t_lane + T_S + 32 * C::CPW * wg + cc * 16, pd);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(TBAR(B_PF));
    }
    if (ok) {
      ok = mbar_wait(TBAR(B_ACC), 0, abort_flag, tmo, ecode | 6);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      using OutT = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
      const bool any = n_jt > 0;
      const size_t o = (static_cast<size_t>(q0 + row) * p.hq + h) * p.dh;
      // group w writes its share of the D columns of dQ (groups past D/32 write none)
      constexpr int CHQ = (D / 32) / C::NWG > 0 ? (D / 32) / C::NWG : 1;
#pragma unroll 1
      for (int c = wg * CHQ; c < (wg + 1) * CHQ && c < D / 32; ++c) {
        uint32_t a[32];
        tmem_ld32(t_lane + T_DQ + c * 32, a);
        tmem_wait_ld();
        if (row < lq) {
          uint32_t pa[16];
#pragma unroll
          for (int u = 0; u < 16; ++u)
            pa[u] = any ? bpack2<BF16>(__uint_as_float(a[2 * u]) * p.scale,
                                       __uint_as_float(a[2 * u + 1]) * p.scale)
                        : 0u;
          uint4* dqp = reinterpret_cast<uint4*>(reinterpret_cast<OutT*>(p.dq) + o + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (c * 32 + u * 8 < p.dh)
              dqp[u] = make_uint4(pa[4 * u], pa[4 * u + 1], pa[4 * u + 2], pa[4 * u + 3]);
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

}  // namespace mea
