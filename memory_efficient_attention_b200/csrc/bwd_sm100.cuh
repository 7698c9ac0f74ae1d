// bwd_sm100.cuh — parameters of the backward pass and its first kernel.
//
// The backward computes dq, dk, dv of L = sum(out * dout) for the forward's definition; its
// main kernels (tcgen05) are in bwd_tc_sm100.cuh. This file holds the parameter block and
//   mea_bwd_pre_kernel   per (query head, token) row, one warp per token over its heads
//                        (HBM-bound: reads out and dout once, in whole 128-byte lines at full
//                        width): nd = -rowsum(dO * O) = -delta and the row's exponent term
//                        na = -lse log2 e (causal ALiBi: also - slope log2 e ((t - q0) mod 32),
//                        t - q0 the row's index in its segment), both fp32 in the workspace.
//                        128 zero rows per head follow the last token, so the tile loops of
//                        the dK/dV kernel may read row terms up to a tile past a segment's end.
//                        Its first block also ranks the segments by decreasing lq + lk (up to
//                        kBwdOrderMax of them): the two main kernels launch the segments in
//                        that order, so the heaviest CTAs start first instead of forming a tail.
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
  float* nd;            // [Hq, t_pad] workspace: -delta of each row (zero in the pad rows)
  float* na;            // [Hq, t_pad] workspace: the row's exponent term (see the pre kernel)
  int t_pad;            // total_q + 128
  int lin_bias;         // causal ALiBi: na carries -slope log2 e ((t - q0) mod 32)
  int* order;           // [n_seqs] workspace: segments by decreasing lq + lk, or null (identity)
  const int32_t* cu_q;
  const int32_t* cu_k;
  const float* slopes;  // [Hq] natural-log ALiBi slopes, or null
  int n_seqs;
  int total_q;
  int total_k;
  int hq;
  int hkv;
  int dh;               // head dim of the rows (<= D; the TMA zero-fills the columns past it)
  int R;                // query heads per KV head
  int mq;               // query heads per dQ CTA (divides hq)
  float scale;
  float c1;             // scale * log2(e)
};

// ------------------------------------------------------------------------------------------
constexpr int kBwdOrderMax = 1024;
// pre kernel, full-width rows: heads covered by one 512-byte warp load, and loads of each of
// out and dout a lane keeps in flight (two: 40 registers, 48 warps per SM; four loads need 64
// registers and run slower at 32 warps per SM)
template <int D>
constexpr int kPreHeadsPerLoad = 256 / D;
constexpr int kPreBatch = 2;

// sum of the eight products of two 16-byte groups of 16-bit values, in fp32
template <bool BF16>
__device__ __forceinline__ float pre_dot8(const uint4 a, const uint4 b) {
  const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    float2 af, bf;
    if constexpr (BF16) {
      af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[u]));
      bf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw[u]));
    } else {
      af = __half22float2(*reinterpret_cast<const __half2*>(&aw[u]));
      bf = __half22float2(*reinterpret_cast<const __half2*>(&bw[u]));
    }
    acc = fmaf(af.x, bf.x, acc);
    acc = fmaf(af.y, bf.y, acc);
  }
  return acc;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(128) mea_bwd_pre_kernel(const BwdParams p) {
  if (blockIdx.x == 0 && p.order) {
    // rank of segment i = number of segments heavier than it (ties by index): a stable sort
    __shared__ int len[kBwdOrderMax];
    for (int i = threadIdx.x; i < p.n_seqs; i += blockDim.x)
      len[i] = (__ldg(p.cu_q + i + 1) - __ldg(p.cu_q + i)) + (__ldg(p.cu_k + i + 1) - __ldg(p.cu_k + i));
    __syncthreads();
    for (int i = threadIdx.x; i < p.n_seqs; i += blockDim.x) {
      const int li = len[i];
      int r = 0;
      for (int j = 0; j < p.n_seqs; ++j) {
        const int lj = len[j];
        r += (lj > li || (lj == li && j < i)) ? 1 : 0;
      }
      p.order[r] = i;
    }
  }
  // One warp per token (four per block): the token's segment is found once, and the rows of
  // its heads, adjacent in memory, are read by the lanes together.
  const int t = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= p.t_pad) return;
  if (t >= p.total_q) {  // pad rows
    for (int h = lane; h < p.hq; h += 32) {
      p.nd[static_cast<size_t>(h) * p.t_pad + t] = 0.f;
      p.na[static_cast<size_t>(h) * p.t_pad + t] = 0.f;
    }
    return;
  }
  constexpr float LOG2E = 1.4426950408889634f;
  int e_row = 0;  // the token's index in its segment, mod 32 (causal ALiBi only)
  if (p.lin_bias) {
    if (lane == 0) {
      // start of the token's segment: the last s with cu_q[s] <= t
      int lo = 0, hi = p.n_seqs;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.cu_q + mid) <= t) lo = mid; else hi = mid;
      }
      e_row = (t - __ldg(p.cu_q + lo)) & 31;
    }
    e_row = __shfl_sync(0xffffffffu, e_row, 0);
  }
  const float* lse_t = p.lse + t;
  if (p.dh == D && p.hq % kPreHeadsPerLoad<D> == 0) {
    // Full-width rows: a head's row spans D/8 adjacent lanes, so every warp load reads 512
    // contiguous bytes (whole 128-byte lines, each sector once); the row sums are reduced
    // over those lanes with shuffles. kPreBatch loads of out and dout are in flight per lane.
    constexpr int LPH = D / 8;
    constexpr int HPL = kPreHeadsPerLoad<D>;
    const size_t row0 = static_cast<size_t>(t) * p.hq * D;
    const uint4* o4 = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.out) + row0) + lane;
    const uint4* g4 = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.dout) + row0) + lane;
    const int n_ld = p.hq / HPL;
    for (int i0 = 0; i0 < n_ld; i0 += kPreBatch) {
      uint4 ov[kPreBatch], gv[kPreBatch];
#pragma unroll
      for (int b = 0; b < kPreBatch; ++b)
        if (i0 + b < n_ld) {
          ov[b] = __ldg(o4 + (i0 + b) * 32);
          gv[b] = __ldg(g4 + (i0 + b) * 32);
        }
#pragma unroll
      for (int b = 0; b < kPreBatch; ++b) {
        if (i0 + b >= n_ld) break;
        float acc = pre_dot8<BF16>(ov[b], gv[b]);
#pragma unroll
        for (int o = LPH / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane % LPH == 0) {
          const int h = (i0 + b) * HPL + lane / LPH;
          const size_t wi = static_cast<size_t>(h) * p.t_pad + t;
          float na = -__ldg(lse_t + static_cast<size_t>(h) * p.total_q) * LOG2E;
          if (p.lin_bias) na = fmaf(-__ldg(p.slopes + h) * LOG2E, static_cast<float>(e_row), na);
          p.nd[wi] = -acc;
          p.na[wi] = na;
        }
      }
    }
    return;
  }
  // Other widths: lane h takes head h (and h + 32, ...), the whole row dot product from
  // 16-byte read-only loads.
  for (int h = lane; h < p.hq; h += 32) {
    const size_t base = (static_cast<size_t>(t) * p.hq + h) * p.dh;
    const uint4* o4 = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.out) + base);
    const uint4* g4 = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.dout) + base);
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      if (c * 8 >= p.dh) break;
      const uint4 ov = __ldg(o4 + c), gv = __ldg(g4 + c);
      const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float2 of, gf;
        if constexpr (BF16) {
          of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[u]));
          gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[u]));
        } else {
          of = __half22float2(*reinterpret_cast<const __half2*>(&ow[u]));
          gf = __half22float2(*reinterpret_cast<const __half2*>(&gw[u]));
        }
        acc = fmaf(of.x, gf.x, acc);
        acc = fmaf(of.y, gf.y, acc);
      }
    }
    const size_t wi = static_cast<size_t>(h) * p.t_pad + t;
    float na = -__ldg(lse_t + static_cast<size_t>(h) * p.total_q) * LOG2E;
    if (p.lin_bias) na = fmaf(-__ldg(p.slopes + h) * LOG2E, static_cast<float>(e_row), na);
    p.nd[wi] = -acc;
    p.na[wi] = na;
  }
}

}  // namespace mea
