// bwd_sm100.cuh — backward pass of exact attention for sm_100a: dq, dk, dv of
// L = sum(out * dout), given q, k, v, out, the forward's lse and dout (packed varlen,
// block-diagonal, bottom-right causal, GQA, ALiBi — the same definition as the forward).
//
// The derivative of the forward definition, per segment and query head h (KV head g = h / R):
//   P = exp(S - lse) with S = scale*QK^T + bias, masked entries 0;
//   delta_i = rowsum(dO_i * O_i);   dS = P * (dO V^T - delta);
//   dV_g += P^T dO;   dK_g += scale * dS^T Q;   dQ = scale * dS K.
// ("How to Build Memory-Efficient Transformers with xFormers…", section "效能對比" times the
// forward and backward of this attention; the formulas are the calculus of the forward.)
//
// Three kernels, no atomics, deterministic:
//   mea_bwd_pre_kernel   delta[h, t] = rowsum(dO * O) in fp32 (one warp per row).
//   mea_bwd_dkdv_kernel  one CTA per (key tile of 64, segment, KV head): loops over the R query
//                        heads of the group and every query tile that sees the key tile; dK, dV
//                        of the tile accumulate in registers across the whole group.
//   mea_bwd_dq_kernel    one CTA per (query tile of 64, segment, query head): loops over the key
//                        tiles the tile sees; dQ accumulates in registers.
// Both main kernels recompute S and dP (the dq kernel twice-over work is the price of having no
// fp32 dq accumulation buffer and no atomics). Tiles are 64 x 64 on warp-level mma.sync
// m16n8k16 with fp32 accumulation: four warps, each owning 16 keys (dkdv) or 16 rows (dq).
// Operands stream through shared memory with cp.async into 128-byte-swizzled tiles read by
// ldmatrix; P and dS are reused from the accumulator registers as A operands.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace mea {

struct BwdParams {
  const void* q;
  const void* k;
  const void* v;
  const void* out;
  const float* lse;     // [Hq, T_q], natural log (the forward's output)
  const void* dout;
  void* dq;
  void* dk;
  void* dv;
  float* delta;         // [Hq, T_q] workspace
  const int32_t* cu_q;
  const int32_t* cu_k;
  const float* slopes;  // [Hq] natural-log ALiBi slopes, or null
  int n_seqs;
  int total_q;
  int total_k;
  int hq;
  int hkv;
  int R;                // query heads per KV head
  float scale;
  float c1;             // scale * log2(e)
};

template <int D>
struct BwdCfg {
  static constexpr int TILE = 64 * D * 2;  // bytes of one [64][D] 16-bit tile
  // six tiles + [2][64] lse and [2][64] delta floats + up to 1 KB of alignment pad
  static constexpr int SMEM = 6 * TILE + 1024 + 1024;
  static constexpr int NT = D / 8;         // 8-column accumulator tiles along D
};

// Byte offset of 16-byte chunk `ch` (0 .. D/8-1) of row `row` in a [64][D] tile stored as D/64
// atoms of [64 rows][128 B], chunks XOR-swizzled by row & 7 so that ldmatrix is conflict-free.
__device__ __forceinline__ uint32_t btile_off(int row, int ch) {
  return static_cast<uint32_t>((ch >> 3) * (64 * 128) + row * 128 + (((ch & 7) ^ (row & 7)) << 4));
}

// cp.async of rows [0, 64) of a [64][D] tile whose row r starts at base + r*stride (elements);
// rows >= nrows are zero-filled.
template <int D>
__device__ __forceinline__ void btile_load(uint32_t sdst, const uint16_t* base, size_t stride,
                                           int nrows, int tid) {
  constexpr int CH = D / 8;
#pragma unroll 4
  for (int i = tid; i < 64 * CH; i += 128) {
    const int row = i / CH, ch = i % CH;
    const bool ok = row < nrows;
    const uint16_t* src = base + (ok ? static_cast<size_t>(row) * stride : 0) + ch * 8;
    cp_async16(sdst + btile_off(row, ch), src, ok ? 16u : 0u);
  }
}

// acc[16 x 64] (8 n-tiles) += A[16 rows of tile sa starting at a_row0] * B^T where B is the
// [64][D] tile sb (rows = n): the product of two row-major tiles over their D columns.
template <int D, bool BF16>
__device__ __forceinline__ void bwd_mm_rows_x_rows(float (&acc)[8][4], uint32_t sa, int a_row0,
                                                   uint32_t sb, int lane) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4(sa + btile_off(a_row0 + (lane & 7) + ((lane >> 3) & 1) * 8, kk * 2 + (lane >> 4)),
            a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sb + btile_off(np * 16 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)),
              b0, b1, b2, b3);
      mma16816<BF16>(acc[2 * np], a, b0, b1);
      mma16816<BF16>(acc[2 * np + 1], a, b2, b3);
    }
  }
}

// out[16 x D] += X[16 x 64] * T[64 x D], X given as accumulator registers (8 n-tiles of 16 x 8,
// packed to 16-bit A fragments here), T the [64][D] tile st read transposed by ldmatrix.
template <int D, bool BF16>
__device__ __forceinline__ void bwd_mm_regs_x_tile(float (&out)[D / 8][4], const float (&x)[8][4],
                                                   uint32_t st, int lane) {
#pragma unroll
  for (int kb = 0; kb < 4; ++kb) {
    uint32_t a[4];
    a[0] = dpack2<BF16>(x[2 * kb][0], x[2 * kb][1]);
    a[1] = dpack2<BF16>(x[2 * kb][2], x[2 * kb][3]);
    a[2] = dpack2<BF16>(x[2 * kb + 1][0], x[2 * kb + 1][1]);
    a[3] = dpack2<BF16>(x[2 * kb + 1][2], x[2 * kb + 1][3]);
#pragma unroll
    for (int nd = 0; nd < D / 16; ++nd) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(st + btile_off(kb * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, nd * 2 + (lane >> 4)),
                b0, b1, b2, b3);
      mma16816<BF16>(out[2 * nd], a, b0, b1);
      mma16816<BF16>(out[2 * nd + 1], a, b2, b3);
    }
  }
}

// ------------------------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(128) mea_bwd_pre_kernel(const BwdParams p) {
  const long long row = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(p.total_q) * p.hq) return;
  const int t = static_cast<int>(row / p.hq), h = static_cast<int>(row % p.hq);
  constexpr int E = D / 32;  // elements per lane
  const size_t base = (static_cast<size_t>(t) * p.hq + h) * D + lane * E;
  const uint16_t* o = reinterpret_cast<const uint16_t*>(p.out) + base;
  const uint16_t* g = reinterpret_cast<const uint16_t*>(p.dout) + base;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    const uint32_t ov = *reinterpret_cast<const uint32_t*>(o + e);
    const uint32_t gv = *reinterpret_cast<const uint32_t*>(g + e);
    float o0, o1, g0, g1;
    if constexpr (BF16) {
      const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov));
      const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv));
      o0 = of.x; o1 = of.y; g0 = gf.x; g1 = gf.y;
    } else {
      const float2 of = __half22float2(*reinterpret_cast<const __half2*>(&ov));
      const float2 gf = __half22float2(*reinterpret_cast<const __half2*>(&gv));
      o0 = of.x; o1 = of.y; g0 = gf.x; g1 = gf.y;
    }
    acc = fmaf(o0, g0, acc);
    acc = fmaf(o1, g1, acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) p.delta[static_cast<size_t>(h) * p.total_q + t] = acc;
}

// ------------------------------------------------------------------------------------------
template <int D, bool BF16, bool CAUSAL, bool ALIBI>
__global__ void __launch_bounds__(128) mea_bwd_dkdv_kernel(const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr float LOG2E = 1.4426950408889634f;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sb = smem_u32(smem);
  const uint32_t sK = sb, sV = sb + C::TILE;
  // buffers b = 0, 1: Q at sb + (2 + 2b) * TILE, dO at sb + (3 + 2b) * TILE
  float* sL = reinterpret_cast<float*>(smem + 6 * C::TILE);  // [2][64] lse * log2(e)
  float* sDl = sL + 128;                                     // [2][64] delta

  const int jt = blockIdx.x, s = blockIdx.y, g = blockIdx.z;
  const int q0 = __ldg(p.cu_q + s), lq = __ldg(p.cu_q + s + 1) - q0;
  const int k0 = __ldg(p.cu_k + s), lk = __ldg(p.cu_k + s + 1) - k0;
  const int key0 = jt * 64;
  if (key0 >= lk) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, t4 = lane & 3;
  const int shift = lk - lq;  // key position of query row i is i + shift (bottom-right)
  const int nkeys = min(64, lk - key0);
  const size_t kv_stride = static_cast<size_t>(p.hkv) * D;
  const size_t q_stride = static_cast<size_t>(p.hq) * D;
  btile_load<D>(sK, reinterpret_cast<const uint16_t*>(p.k) + (static_cast<size_t>(k0 + key0) * p.hkv + g) * D,
                kv_stride, nkeys, tid);
  btile_load<D>(sV, reinterpret_cast<const uint16_t*>(p.v) + (static_cast<size_t>(k0 + key0) * p.hkv + g) * D,
                kv_stride, nkeys, tid);
  // Query tiles that see at least one key of this tile (causal: rows with i + shift >= key0).
  const int it0 = CAUSAL ? max(0, key0 - shift) / 64 : 0;
  const int n_it = (lq + 63) / 64;
  const int nt = n_it - it0;
  const int n_iter = nt > 0 ? nt * p.R : 0;

  auto issue = [&](int t, int buf) {
    const int r = t / nt, it = it0 + t % nt;
    const int h = g * p.R + r;
    const int row0 = it * 64, nrows = min(64, lq - row0);
    const size_t off = (static_cast<size_t>(q0 + row0) * p.hq + h) * D;
    btile_load<D>(sb + (2 + 2 * buf) * C::TILE, reinterpret_cast<const uint16_t*>(p.q) + off,
                  q_stride, nrows, tid);
    btile_load<D>(sb + (3 + 2 * buf) * C::TILE, reinterpret_cast<const uint16_t*>(p.dout) + off,
                  q_stride, nrows, tid);
    if (tid < 64) {
      const bool ok = tid < nrows;
      const size_t li = static_cast<size_t>(h) * p.total_q + q0 + row0 + tid;
      sL[buf * 64 + tid] = ok ? __ldg(p.lse + li) * LOG2E : 0.f;
      sDl[buf * 64 + tid] = ok ? p.delta[li] : 0.f;
    }
  };

  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;

  if (n_iter > 0) issue(0, 0);
  cp_async_commit();
  for (int t = 0; t < n_iter; ++t) {
    const int buf = t & 1;
    if (t + 1 < n_iter) issue(t + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sQ = sb + (2 + 2 * buf) * C::TILE, sdO = sb + (3 + 2 * buf) * C::TILE;
    const int r = t / nt, it = it0 + t % nt;
    const int h = g * p.R + r;
    const int row0 = it * 64;
    float slope2 = 0.f;
    if constexpr (ALIBI) slope2 = __ldg(p.slopes + h) * LOG2E;
    // ---- S^T (16 keys of this warp x 64 rows) and P^T
    float x[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) x[n][e] = 0.f;
    bwd_mm_rows_x_rows<D, BF16>(x, sK, warp * 16, sQ, lane);
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = key0 + warp * 16 + gid + (e >> 1) * 8;
        const int rl = n * 8 + 2 * t4 + (e & 1);
        const int i = row0 + rl;
        const bool valid = i < lq && key < lk && (!CAUSAL || key <= i + shift);
        float z = x[n][e] * p.c1 - sL[buf * 64 + rl];
        if constexpr (ALIBI) z -= slope2 * fabsf(static_cast<float>(i + shift - key));
        x[n][e] = valid ? ex2_approx(z) : 0.f;
      }
    // ---- dV += P^T dO
    bwd_mm_regs_x_tile<D, BF16>(dv, x, sdO, lane);
    // ---- dP^T = V dO^T, dS^T = P^T * (dP^T - delta)
    float y[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) y[n][e] = 0.f;
    bwd_mm_rows_x_rows<D, BF16>(y, sV, warp * 16, sdO, lane);
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int rl = n * 8 + 2 * t4 + (e & 1);
        x[n][e] = x[n][e] * (y[n][e] - sDl[buf * 64 + rl]);
      }
    // ---- dK += dS^T Q (scaled at the end)
    bwd_mm_regs_x_tile<D, BF16>(dk, x, sQ, lane);
    __syncthreads();
  }
  cp_async_wait<0>();
  // ---- write dK (scaled), dV for the keys of this tile
  using OutT = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int kl = warp * 16 + gid + hf * 8;
      if (key0 + kl < lk) {
        const size_t o = (static_cast<size_t>(k0 + key0 + kl) * p.hkv + g) * D + n * 8 + 2 * t4;
        *reinterpret_cast<uint32_t*>(reinterpret_cast<OutT*>(p.dk) + o) =
            dpack2<BF16>(dk[n][2 * hf] * p.scale, dk[n][2 * hf + 1] * p.scale);
        *reinterpret_cast<uint32_t*>(reinterpret_cast<OutT*>(p.dv) + o) =
            dpack2<BF16>(dv[n][2 * hf], dv[n][2 * hf + 1]);
      }
    }
}

// ------------------------------------------------------------------------------------------
template <int D, bool BF16, bool CAUSAL, bool ALIBI>
__global__ void __launch_bounds__(128) mea_bwd_dq_kernel(const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr float LOG2E = 1.4426950408889634f;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb, sdO = sb + C::TILE;
  // buffers b = 0, 1: K at sb + (2 + 2b) * TILE, V at sb + (3 + 2b) * TILE

  // Causal: the last query tiles see the most keys; start them first.
  const int itile = CAUSAL ? static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x)
                           : static_cast<int>(blockIdx.x);
  const int s = blockIdx.y, h = blockIdx.z, g = h / p.R;
  const int q0 = __ldg(p.cu_q + s), lq = __ldg(p.cu_q + s + 1) - q0;
  const int k0 = __ldg(p.cu_k + s), lk = __ldg(p.cu_k + s + 1) - k0;
  const int row0 = itile * 64;
  if (row0 >= lq) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, t4 = lane & 3;
  const int shift = lk - lq;
  const int nrows = min(64, lq - row0);
  const size_t q_stride = static_cast<size_t>(p.hq) * D;
  const size_t kv_stride = static_cast<size_t>(p.hkv) * D;
  const size_t qoff = (static_cast<size_t>(q0 + row0) * p.hq + h) * D;
  btile_load<D>(sQ, reinterpret_cast<const uint16_t*>(p.q) + qoff, q_stride, nrows, tid);
  btile_load<D>(sdO, reinterpret_cast<const uint16_t*>(p.dout) + qoff, q_stride, nrows, tid);
  // Per-row values of the two rows this thread holds (rows warp*16 + gid, + 8).
  float lse2[2], dl[2];
  int irow[2];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int i = row0 + warp * 16 + gid + hf * 8;
    irow[hf] = i;
    const size_t li = static_cast<size_t>(h) * p.total_q + q0 + i;
    lse2[hf] = i < lq ? __ldg(p.lse + li) * LOG2E : 0.f;
    dl[hf] = i < lq ? p.delta[li] : 0.f;
  }
  float slope2 = 0.f;
  if constexpr (ALIBI) slope2 = __ldg(p.slopes + h) * LOG2E;
  // Key tiles seen by this query tile.
  int n_jt = (lk + 63) / 64;
  if (CAUSAL) {
    const int kmax = min(lk - 1, row0 + nrows - 1 + shift);
    n_jt = kmax >= 0 ? kmax / 64 + 1 : 0;
  }
  auto issue = [&](int jt, int buf) {
    const int nk = min(64, lk - jt * 64);
    const size_t off = (static_cast<size_t>(k0 + jt * 64) * p.hkv + g) * D;
    btile_load<D>(sb + (2 + 2 * buf) * C::TILE, reinterpret_cast<const uint16_t*>(p.k) + off,
                  kv_stride, nk, tid);
    btile_load<D>(sb + (3 + 2 * buf) * C::TILE, reinterpret_cast<const uint16_t*>(p.v) + off,
                  kv_stride, nk, tid);
  };
  float dq[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[i][e] = 0.f;
  if (n_jt > 0) issue(0, 0);
  cp_async_commit();
  for (int jt = 0; jt < n_jt; ++jt) {
    const int buf = jt & 1;
    if (jt + 1 < n_jt) issue(jt + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sK = sb + (2 + 2 * buf) * C::TILE, sV = sb + (3 + 2 * buf) * C::TILE;
    // ---- S (16 rows of this warp x 64 keys) and P
    float x[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) x[n][e] = 0.f;
    bwd_mm_rows_x_rows<D, BF16>(x, sQ, warp * 16, sK, lane);
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hf = e >> 1;
        const int key = jt * 64 + n * 8 + 2 * t4 + (e & 1);
        const int i = irow[hf];
        const bool valid = i < lq && key < lk && (!CAUSAL || key <= i + shift);
        float z = x[n][e] * p.c1 - lse2[hf];
        if constexpr (ALIBI) z -= slope2 * fabsf(static_cast<float>(i + shift - key));
        x[n][e] = valid ? ex2_approx(z) : 0.f;
      }
    // ---- dP = dO V^T, dS = P * (dP - delta)
    float y[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) y[n][e] = 0.f;
    bwd_mm_rows_x_rows<D, BF16>(y, sdO, warp * 16, sV, lane);
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) x[n][e] = x[n][e] * (y[n][e] - dl[e >> 1]);
    // ---- dQ += dS K (scaled at the end)
    bwd_mm_regs_x_tile<D, BF16>(dq, x, sK, lane);
    __syncthreads();
  }
  cp_async_wait<0>();
  using OutT = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int i = irow[hf];
      if (i < lq) {
        const size_t o = (static_cast<size_t>(q0 + i) * p.hq + h) * D + n * 8 + 2 * t4;
        *reinterpret_cast<uint32_t*>(reinterpret_cast<OutT*>(p.dq) + o) =
            dpack2<BF16>(dq[n][2 * hf] * p.scale, dq[n][2 * hf + 1] * p.scale);
      }
    }
}

}  // namespace mea
