// mea_api.cu — the C ABI of libmea (declared in include/mea.h): argument validation, TMA
// descriptor encoding and kernel launches. No device memory is allocated here; no call
// synchronises the host except mea_device_error.
#include <cudaTypedefs.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/mea.h"
#include "bwd_sm100.cuh"
#include "bwd_tc_sm100.cuh"
#include "decode_sm100.cuh"
#include "fwd256_sm100.cuh"
#include "fwd_sm100.cuh"
#include "ptx.cuh"

namespace {

std::atomic<unsigned long long> g_timeout_ns{2000000000ull};

struct DeviceInfo {
  bool init = false;
  bool ok = false;
  int sms = 0;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device_info(DeviceInfo& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MEA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MEA_ERR_CUDA;
    d.ok = (major == 10);
    d.sms = sms;
    d.init = true;
  }
  out = d;
  return d.ok ? MEA_OK : MEA_ERR_DEVICE;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }();
  return fn;
}

// 3-D tiled map over a row-major [d2, d1, d0] tensor of 16-bit elements, 128-byte swizzle.
constexpr int kDtypeE4M3 = 2;  // internal: 8-bit e4m3 tensor (mea_forward_fp8)

bool encode_3d_uncached(CUtensorMap* map, const void* base, int dtype, uint64_t d0,
                        uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t es = dtype == kDtypeE4M3 ? 1 : 2;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * es, d0 * d1 * es};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, dtype == kDtypeE4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                       : dtype == MEA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                  3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------------------------------
// Cache of encoded tensor maps. A map only describes (address, sizes, strides, box, element
// type, swizzle), so one encoded for the same arguments is the same 128 bytes; serving calls
// that reuse their buffers (every decode step of a KV cache, for instance) skip the encoding.
// The cache is the library's only state besides per-device attributes: kMapCache entries,
// least recently used replaced first, guarded by a mutex.
// ------------------------------------------------------------------------------------------
struct MapKey {
  const void* base;
  int dtype, rank;
  uint64_t dims[5];
  uint32_t box[5];
  bool operator==(const MapKey& o) const {
    if (base != o.base || dtype != o.dtype || rank != o.rank) return false;
    for (int i = 0; i < 5; ++i)
      if (dims[i] != o.dims[i] || box[i] != o.box[i]) return false;
    return true;
  }
};
constexpr int kMapCache = 64;
struct MapCache {
  MapKey key[kMapCache];
  CUtensorMap map[kMapCache];
  uint64_t used[kMapCache] = {};  // 0 = empty slot
  uint64_t tick = 0;
  std::mutex mu;
};
MapCache g_maps;

// Copies the cached map for `k` into *out; false when it is not cached.
bool map_lookup(const MapKey& k, CUtensorMap* out) {
  std::lock_guard<std::mutex> lk(g_maps.mu);
  for (int i = 0; i < kMapCache; ++i)
    if (g_maps.used[i] && g_maps.key[i] == k) {
      g_maps.used[i] = ++g_maps.tick;
      *out = g_maps.map[i];
      return true;
    }
  return false;
}

void map_insert(const MapKey& k, const CUtensorMap& m) {
  std::lock_guard<std::mutex> lk(g_maps.mu);
  int victim = 0;
  for (int i = 0; i < kMapCache; ++i) {
    if (g_maps.used[i] == 0) {
      victim = i;
      break;
    }
    if (g_maps.used[i] < g_maps.used[victim]) victim = i;
  }
  g_maps.key[victim] = k;
  g_maps.map[victim] = m;
  g_maps.used[victim] = ++g_maps.tick;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Head dims of the forward: a multiple of 8 from 8 to 128 for 16-bit inputs (16-byte rows), a
// multiple of 16 from 16 to 128 for e4m3 inputs.
// Head dims from 136 to 256 (16-bit only) run in the 256-wide kernel.
bool fwd_head_dim_ok(int d, bool e8) {
  return e8 ? (d >= 16 && d <= 128 && d % 16 == 0) : (d >= 8 && d <= 256 && d % 8 == 0);
}

int largest_pow2_divisor(int x, int cap) {
  int p = 1;
  while (p * 2 <= cap && x % (p * 2) == 0) p *= 2;
  return p;
}

// Shifts for the power-of-two packing factors and the multiplier that maps a head block to its
// KV group (see FwdParams). Returns false when (hb * g_mul) >> 32 would not be exact for every
// head block ((n_hb - 1) * (d - 1) < 2^32 is sufficient).
static bool fwd_schedule_constants(mea::FwdParams& p) {
  int l2p = 0;
  while ((1 << l2p) < p.P) ++l2p;
  int l2t = 0;
  while ((1 << l2t) < p.subtiles * p.tok_per_tile) ++l2t;
  p.log2_p = l2p;
  p.log2_tpp = l2t;
  const unsigned long long d = static_cast<unsigned long long>(p.R / p.P);
  p.g_mul = ((1ull << 32) + d - 1) / d;
  return static_cast<unsigned long long>(p.n_hb - 1) * (d - 1) < (1ull << 32);
}

// cudaFuncSetAttribute(max dynamic shared memory) once per (kernel, device); the result of that
// one call is kept and returned on every later call, so a failure is never forgotten. The kernel
// is a template argument so that every kernel (not every kernel signature) has its own state.
template <auto kern>
cudaError_t smem_attr_once(uint32_t smem) {
  static std::once_flag once[kMaxDevices];
  static cudaError_t result[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    result[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  return result[dev];
}

// Drops a launch error left by an earlier, unrelated call, so that the check after this
// call's launches reports only their own failures.
inline void clear_stale_launch_error() { (void)cudaGetLastError(); }

// ------------------------------------------------------------------------------------------
// Forward launch dispatch.
// ------------------------------------------------------------------------------------------
template <int D, bool BF16, bool CAUSAL, bool ALIBI, bool E8 = false>
int launch_fwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const CUtensorMap& to, const mea::FwdParams& p, int grid, cudaStream_t stream) {
  constexpr auto kern = mea::mea_fwd_sm100_kernel<D, BF16, CAUSAL, ALIBI, E8>;
  constexpr uint32_t smem = mea::FwdCfg<D, E8>::SMEM_TOTAL;
  if (smem_attr_once<kern>(smem) != cudaSuccess) return MEA_ERR_CUDA;
  clear_stale_launch_error();
  kern<<<grid, mea::FwdCfg<D>::THREADS, smem, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError() == cudaSuccess ? MEA_OK : MEA_ERR_CUDA;
}

template <bool BF16, bool CAUSAL, bool ALIBI>
int launch_fwd256_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const mea::FwdParams& p, int grid, cudaStream_t stream) {
  constexpr auto kern = mea::mea_fwd256_sm100_kernel<BF16, CAUSAL, ALIBI>;
  constexpr uint32_t smem = mea::Fwd256Cfg::SMEM_TOTAL;
  if (smem_attr_once<kern>(smem) != cudaSuccess) return MEA_ERR_CUDA;
  clear_stale_launch_error();
  kern<<<grid, mea::Fwd256Cfg::THREADS, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? MEA_OK : MEA_ERR_CUDA;
}

template <bool BF16>
int launch_fwd256_d(bool causal, bool alibi, const CUtensorMap& tq, const CUtensorMap& tk,
                    const CUtensorMap& tv, const mea::FwdParams& p, int grid, cudaStream_t s) {
  if (causal)
    return alibi ? launch_fwd256_t<BF16, true, true>(tq, tk, tv, p, grid, s)
                 : launch_fwd256_t<BF16, true, false>(tq, tk, tv, p, grid, s);
  return alibi ? launch_fwd256_t<BF16, false, true>(tq, tk, tv, p, grid, s)
               : launch_fwd256_t<BF16, false, false>(tq, tk, tv, p, grid, s);
}

template <int D, bool BF16, bool E8 = false>
int launch_fwd_d(bool causal, bool alibi, const CUtensorMap& tq, const CUtensorMap& tk,
                 const CUtensorMap& tv, const CUtensorMap& to, const mea::FwdParams& p, int grid,
                 cudaStream_t s) {
  if (causal)
    return alibi ? launch_fwd_t<D, BF16, true, true, E8>(tq, tk, tv, to, p, grid, s)
                 : launch_fwd_t<D, BF16, true, false, E8>(tq, tk, tv, to, p, grid, s);
  return alibi ? launch_fwd_t<D, BF16, false, true, E8>(tq, tk, tv, to, p, grid, s)
               : launch_fwd_t<D, BF16, false, false, E8>(tq, tk, tv, to, p, grid, s);
}


// 3-D / 4-D maps through the cache (same arguments as the uncached encoders).
bool encode_3d(CUtensorMap* map, const void* base, int dtype, uint64_t d0, uint64_t d1,
               uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2) {
  const MapKey k{base, dtype, 3, {d0, d1, d2, 0}, {b0, b1, b2, 0}};
  if (map_lookup(k, map)) return true;
  if (!encode_3d_uncached(map, base, dtype, d0, d1, d2, b0, b1, b2)) return false;
  map_insert(k, *map);
  return true;
}

// 4-D tiled map over a paged cache [d3 blocks, d2 slots, d1 heads, d0] of 16-bit elements.
bool encode_4d_uncached(CUtensorMap* map, const void* base, int dtype, uint64_t d0,
                        uint64_t d1, uint64_t d2, uint64_t d3, uint32_t b0, uint32_t b1,
                        uint32_t b2, uint32_t b3) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
  cuuint32_t box[4] = {b0, b1, b2, b3};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, dtype == MEA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                  4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_4d(CUtensorMap* map, const void* base, int dtype, uint64_t d0, uint64_t d1,
               uint64_t d2, uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  const MapKey k{base, dtype, 4, {d0, d1, d2, d3}, {b0, b1, b2, b3}};
  if (map_lookup(k, map)) return true;
  if (!encode_4d_uncached(map, base, dtype, d0, d1, d2, d3, b0, b1, b2, b3)) return false;
  map_insert(k, *map);
  return true;
}

// 5-D tiled map over a paged cache [blocks, slots, heads, head_dim] of 16-bit elements with
// head_dim = 64 * atoms, seen as (64 columns, slot, atom, head, block): one box {64, rows, atoms,
// 1, 1} brings `rows` slots of one head and block with every 64-column atom, landing as
// [atom][rows][128 B] (the 128-byte swizzle per 128-byte row).
bool encode_paged5(CUtensorMap* map, const void* base, int dtype, uint64_t head_dim,
                   uint64_t heads, uint64_t slots, uint64_t blocks, uint32_t rows) {
  const uint64_t atoms = head_dim / 64;
  const MapKey k{base, dtype, 5, {64, slots, atoms, heads, blocks}, {64, rows, uint32_t(atoms), 1, 1}};
  if (map_lookup(k, map)) return true;
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[5] = {64, slots, atoms, heads, blocks};
  cuuint64_t strides[4] = {heads * head_dim * 2, 128, head_dim * 2, slots * heads * head_dim * 2};
  cuuint32_t box[5] = {64, rows, static_cast<cuuint32_t>(atoms), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, dtype == MEA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                  5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  map_insert(k, *map);
  return true;
}

// ------------------------------------------------------------------------------------------
// Backward launch dispatch.
// ------------------------------------------------------------------------------------------
struct BwdMaps {
  CUtensorMap q, dout, k, v;  // 128-row boxes of one head
};

template <int D, bool BF16, bool CAUSAL, bool ALIBI>
int launch_bwd_t(const BwdMaps& m, const mea::BwdParams& p, int max_q, int max_k,
                 cudaStream_t stream) {
  constexpr uint32_t smem = mea::BwdKvCfg<D>::SMEM_TOTAL;
  constexpr uint32_t smem_dq = mea::BwdDqCfg<D>::SMEM_TOTAL;
  constexpr auto kdkdv = mea::mea_bwd_dkdv_tc_kernel<D, BF16, CAUSAL, ALIBI>;
  constexpr auto kdq = mea::mea_bwd_dq_tc_kernel<D, BF16, CAUSAL, ALIBI>;
  if (smem_attr_once<kdkdv>(smem) != cudaSuccess || smem_attr_once<kdq>(smem_dq) != cudaSuccess)
    return MEA_ERR_CUDA;
  clear_stale_launch_error();
  const unsigned long long tmo = g_timeout_ns.load();
  // one warp per token (including the pad rows), four per block
  mea::mea_bwd_pre_kernel<D, BF16><<<static_cast<unsigned>((p.t_pad + 3) / 4), 128, 0, stream>>>(p);
  if (max_k > 0)
    kdkdv<<<dim3((max_k + 127) / 128, p.n_seqs, p.hkv), mea::BwdTcCfg<D>::THREADS, smem,
            stream>>>(m.q, m.dout, m.k, m.v, p, tmo);
  if (max_q > 0)
    kdq<<<dim3(static_cast<unsigned>((p.hq / p.mq) * ((max_q + 127) / 128)), p.n_seqs),
          mea::BwdTcCfg<D>::THREADS, smem_dq,
          stream>>>(m.q, m.dout, m.k, m.v, p, tmo);
  return cudaGetLastError() == cudaSuccess ? MEA_OK : MEA_ERR_CUDA;
}

template <int D, bool BF16>
int launch_bwd_d(bool causal, bool alibi, const BwdMaps& m, const mea::BwdParams& p, int mq,
                 int mk, cudaStream_t s) {
  if (causal)
    return alibi ? launch_bwd_t<D, BF16, true, true>(m, p, mq, mk, s)
                 : launch_bwd_t<D, BF16, true, false>(m, p, mq, mk, s);
  return alibi ? launch_bwd_t<D, BF16, false, true>(m, p, mq, mk, s)
               : launch_bwd_t<D, BF16, false, false>(m, p, mq, mk, s);
}

// ------------------------------------------------------------------------------------------
// Decode launch dispatch.
// ------------------------------------------------------------------------------------------
template <int D, bool BF16, bool ALIBI, bool PAGED>
int launch_dec_t(const CUtensorMap& tk, const CUtensorMap& tv, const mea::DecParams& p,
                 int grid, int n_kv_heads, cudaStream_t stream) {
  constexpr auto kern = mea::mea_decode_split_kernel<D, BF16, ALIBI, PAGED>;
  constexpr uint32_t smem = mea::DecCfg<D, PAGED>::SMEM_TOTAL;
  if (smem_attr_once<kern>(smem) != cudaSuccess) return MEA_ERR_CUDA;
  clear_stale_launch_error();
  if (grid > 0) kern<<<grid, mea::DecCfg<D, PAGED>::THREADS, smem, stream>>>(tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return MEA_ERR_CUDA;
  dim3 mgrid(p.n_seqs, n_kv_heads);
  mea::mea_lse_merge_kernel<D, BF16><<<mgrid, 256, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? MEA_OK : MEA_ERR_CUDA;
}

template <int D, bool BF16, bool PAGED = false>
int launch_dec_d(bool alibi, const CUtensorMap& tk, const CUtensorMap& tv,
                 const mea::DecParams& p, int grid, int hkv, cudaStream_t s) {
  return alibi ? launch_dec_t<D, BF16, true, PAGED>(tk, tv, p, grid, hkv, s)
               : launch_dec_t<D, BF16, false, PAGED>(tk, tv, p, grid, hkv, s);
}

// Keys per chunk when the caller leaves it to the library: the largest power of two from 128 to
// 2048 that still gives about half a work item (chunk, head block) per SM or more. Every item
// costs a fixed ~1.4 us (its four warps' merge and partial write) beside streaming its keys, so
// few long items beat many short ones: on 64 requests of U[512, 32768] keys 2048-key chunks
// stream at the HBM copy rate where 1024 reach 0.95 of it, and one 32768-key request is 3.4x
// faster at 2048 than at 128, although 2048 leaves 20 of 148 SMs without an item.
int auto_split_keys(int total_k, int n_hb, int sms) {
  long long work = static_cast<long long>(total_k) * n_hb;
  long long target = 2 * work / static_cast<long long>(sms > 0 ? sms : 148);
  int c = 128;
  while (c < 2048 && c * 2 <= target) c *= 2;
  return c;
}

int decode_rb(int R) {
  int rb = 1;
  for (int d = 1; d <= 16; ++d)
    if (R % d == 0) rb = d;
  return rb;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct DecLayout {
  int chunk = 0, n_slots = 0;
  size_t o_bytes = 0, lse_off = 0, total = 0;
};

// Head dims of the decode: a multiple of 8 from 8 to 256; the kernels run 64, 128 or 256 wide.
bool dec_head_dim_ok(int d) { return d >= 8 && d <= 256 && d % 8 == 0; }
int padded_head_dim(int d) { return d <= 64 ? 64 : d <= 128 ? 128 : 256; }

bool dec_layout(int n_seqs, int total_k, int hq, int hkv, int d, int split_keys, int sms,
                DecLayout& L) {
  if (n_seqs < 1 || total_k < 0 || hq < 1 || hkv < 1 || hq % hkv || !dec_head_dim_ok(d))
    return false;
  d = padded_head_dim(d);  // the partials are kept at the kernel's width
  if (split_keys < 0 || split_keys % 64) return false;
  const int R = hq / hkv;
  const int n_hb = hq / decode_rb(R);
  L.chunk = split_keys ? split_keys : auto_split_keys(total_k, n_hb, sms);
  const long long slots = (static_cast<long long>(total_k) + L.chunk - 1) / L.chunk + n_seqs;
  if (slots > (1ll << 30)) return false;
  L.n_slots = static_cast<int>(slots);
  L.o_bytes = static_cast<size_t>(slots) * hq * d * sizeof(float);
  L.lse_off = align_up(L.o_bytes, 256);
  L.total = L.lse_off + align_up(static_cast<size_t>(slots) * hq * sizeof(float), 256);
  return true;
}

}  // namespace

// ------------------------------------------------------------------------------------------
// Fixed scratch for mea_decode_splitkv_noalloc: the split-KV partials live in this array, which
// belongs to the library image (every GPU that loads the library holds it until exit), so that
// callers which cannot allocate device memory can still decode. Host code must not pass the
// symbol itself to a kernel: on the host it is only a stand-in; its device address is looked up
// once per device with cudaGetSymbolAddress.
// ------------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char mea_noalloc_scratch[MEA_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {

PFN_cuCtxGetCurrent_v4000 ctx_current_fn() {
  static PFN_cuCtxGetCurrent_v4000 fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuCtxGetCurrent_v4000>(nullptr);
    return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
  }();
  return fn;
}

// The device address of mea_noalloc_scratch belongs to the CUDA context that was current when
// it was looked up (a device can carry several contexts, and a context can be destroyed and
// recreated). It is cached per device together with that context and looked up again
// whenever a call runs under another one.
struct NoallocAddr {
  CUcontext ctx = nullptr;
  void* addr = nullptr;
};
NoallocAddr g_noalloc[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of mea_noalloc_scratch for the current device and context.
int noalloc_scratch_address(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MEA_ERR_CUDA;
  auto get_ctx = ctx_current_fn();
  if (!get_ctx) return MEA_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return MEA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocAddr& e = g_noalloc[dev];
  if (ctx == nullptr || e.ctx != ctx || e.addr == nullptr) {
    // The lookup makes the device's primary context current when no context is yet.
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, mea_noalloc_scratch) != cudaSuccess || p == nullptr)
      return MEA_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return MEA_ERR_CUDA;
    e.ctx = ctx;
    e.addr = p;
  }
  *ptr = e.addr;
  return MEA_OK;
}

}  // namespace

namespace mea {
// One warp; lane 0 owns the barrier. The wait is the same bounded mbar_wait the kernels use.
__global__ void mea_wait_selftest_kernel(unsigned long long timeout_ns, int arrive) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(b, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    if (arrive) mbar_arrive(b);
    mbar_wait(b, 0, &abort_flag, timeout_ns, MEA_SELFTEST_WAIT_CODE);
  }
  __syncwarp();
}
}  // namespace mea

// dtype: the 16-bit type of out (and of q, k, v unless e8); e8: q, k, v are e4m3 with descales
// qk_descale (folded into the exponent) and v_descale (applied to O before the division by l).
int forward_impl(const void* q, const void* k, const void* v, void* out, float* lse,
                 const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int n_seqs,
                 int total_q, int total_k, int max_seqlen_q, int n_heads_q, int n_heads_kv,
                 int head_dim, float scale, int mask_kind, const float* alibi_slopes, int dtype,
                 bool e8, float qk_descale, float v_descale, void* stream) {
  if (!q || !k || !v || !out || !cu_seqlens_q || !cu_seqlens_k) return MEA_ERR_NULL;
  if (n_seqs < 1 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_q > total_q)
    return MEA_ERR_SHAPE;
  if (n_heads_q < 1 || n_heads_kv < 1 || n_heads_q % n_heads_kv != 0) return MEA_ERR_HEADS;
  // Rows of 16-bit elements need a multiple of 16 bytes (TMA strides); e4m3 rows the same.
  if (!fwd_head_dim_ok(head_dim, e8)) return MEA_ERR_HEAD_DIM;
  if (dtype != MEA_F16 && dtype != MEA_BF16) return MEA_ERR_DTYPE;
  if (mask_kind != MEA_MASK_NONE && mask_kind != MEA_MASK_CAUSAL) return MEA_ERR_MASK;
  if (!std::isfinite(scale) || !std::isfinite(qk_descale) || !std::isfinite(v_descale))
    return MEA_ERR_SCALE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      (lse && !aligned(lse, 4)) || !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4) ||
      (alibi_slopes && !aligned(alibi_slopes, 4)))
    return MEA_ERR_ALIGN;
  DeviceInfo di;
  if (int rc = current_device_info(di); rc != MEA_OK) return rc;
  if (total_q == 0) return MEA_OK;

  const int R = n_heads_q / n_heads_kv;
  const int P = largest_pow2_divisor(R, 128);
  mea::FwdParams p{};
  p.out = out;
  p.lse = lse;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.slopes = alibi_slopes;
  p.n_seqs = n_seqs;
  p.total_q = total_q;
  p.hq = n_heads_q;
  p.dh = head_dim;
  p.P = P;
  p.R = R;
  p.n_hb = n_heads_q / P;
  p.tok_per_tile = 128 / P;
  const bool wide = head_dim > 128;  // one 128-row sub-tile per work item
  p.subtiles = wide ? 1 : 2;
  p.c1 = scale * qk_descale * 1.4426950408889634f;
  p.o_scale = v_descale;
  p.timeout_ns = g_timeout_ns.load();
  if (!fwd_schedule_constants(p)) return MEA_ERR_HEADS;

  CUtensorMap tq, tk, tv, to;
  const uint64_t tk_rows = total_k > 0 ? static_cast<uint64_t>(total_k) : 1;
  const int in_dtype = e8 ? kDtypeE4M3 : dtype;
  const uint32_t box0 = e8 ? 128 : 64;  // elements per 128-byte swizzle row
  // out: one warp's 32 rows (32/P tokens x P heads, or 32 of the P heads of one token).
  const uint32_t out_heads = P < 32 ? static_cast<uint32_t>(P) : 32u;
  const uint32_t out_toks = P < 32 ? static_cast<uint32_t>(32 / P) : 1u;
  if (!encode_3d(&tq, q, in_dtype, head_dim, n_heads_q, total_q, box0, P, 128 / P) ||
      !encode_3d(&tk, k, in_dtype, head_dim, n_heads_kv, tk_rows, box0, 1, 128) ||
      !encode_3d(&tv, v, in_dtype, head_dim, n_heads_kv, tk_rows, box0, 1, 128) ||
      !encode_3d(&to, out, dtype, head_dim, n_heads_q, total_q, 64, out_heads, out_toks))
    return MEA_ERR_CUDA;
  // Every CTA walks the live items of the whole problem; max_seqlen_q only bounds how many
  // can exist, so a grid wider than that would leave CTAs idle.
  const int tok_per_item = p.subtiles * p.tok_per_tile;
  const long long pairs_max =
      (static_cast<long long>(max_seqlen_q) + tok_per_item - 1) / tok_per_item;
  const long long items_max = pairs_max * n_seqs * p.n_hb;
  const int grid = static_cast<int>(items_max < di.sms ? (items_max > 0 ? items_max : 1) : di.sms);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool causal = mask_kind == MEA_MASK_CAUSAL;
  const bool alibi = alibi_slopes != nullptr;
  if (wide)
    return dtype == MEA_BF16 ? launch_fwd256_d<true>(causal, alibi, tq, tk, tv, p, grid, s)
                             : launch_fwd256_d<false>(causal, alibi, tq, tk, tv, p, grid, s);
  if (e8)
    return dtype == MEA_BF16
               ? launch_fwd_d<128, true, true>(causal, alibi, tq, tk, tv, to, p, grid, s)
               : launch_fwd_d<128, false, true>(causal, alibi, tq, tk, tv, to, p, grid, s);
  // Head dims below 64 run in the 64-wide kernel, those up to 128 in the 128-wide one: the TMA
  // loads fill the columns past head_dim with zeros (they add nothing to Q K^T and give zero
  // columns of O, which no store writes).
  if (head_dim > 64)
    return dtype == MEA_BF16 ? launch_fwd_d<128, true>(causal, alibi, tq, tk, tv, to, p, grid, s)
                             : launch_fwd_d<128, false>(causal, alibi, tq, tk, tv, to, p, grid, s);
  return dtype == MEA_BF16 ? launch_fwd_d<64, true>(causal, alibi, tq, tk, tv, to, p, grid, s)
                           : launch_fwd_d<64, false>(causal, alibi, tq, tk, tv, to, p, grid, s);
}

extern "C" {

const char* mea_version(void) { return "mea 0.1.0 (sm_100a)"; }

const char* mea_status_string(int status) {
  switch (status) {
    case MEA_OK: return "MEA_OK: success";
    case MEA_ERR_NULL: return "MEA_ERR_NULL: a required pointer is NULL";
    case MEA_ERR_SHAPE: return "MEA_ERR_SHAPE: invalid sizes";
    case MEA_ERR_HEADS: return "MEA_ERR_HEADS: n_heads_q must be a positive multiple of n_heads_kv";
    case MEA_ERR_HEAD_DIM:
      return "MEA_ERR_HEAD_DIM: head_dim is not supported by this entry point (see mea.h)";
    case MEA_ERR_DTYPE: return "MEA_ERR_DTYPE: dtype must be MEA_F16 or MEA_BF16";
    case MEA_ERR_ALIGN: return "MEA_ERR_ALIGN: tensor base pointers must be 16-byte aligned";
    case MEA_ERR_MASK: return "MEA_ERR_MASK: mask_kind is not a mea_mask value";
    case MEA_ERR_WORKSPACE: return "MEA_ERR_WORKSPACE: workspace missing or too small";
    case MEA_ERR_CUDA: return "MEA_ERR_CUDA: a CUDA call or kernel launch failed";
    case MEA_ERR_DEVICE_TIMEOUT: return "MEA_ERR_DEVICE_TIMEOUT: a kernel gave up on a bounded wait";
    case MEA_ERR_DEVICE: return "MEA_ERR_DEVICE: the current device is not sm_100";
    case MEA_ERR_SCALE: return "MEA_ERR_SCALE: scale must be finite";
    case MEA_ERR_SCRATCH_LIMIT:
      return "MEA_ERR_SCRATCH_LIMIT: the decode partials do not fit in the library's fixed "
             "scratch array (MEA_DECODE_NOALLOC_SCRATCH_BYTES); use mea_decode_splitkv with a "
             "workspace, or a larger split_keys";
    default: return "unknown mea_status";
  }
}

void mea_set_wait_timeout_ns(unsigned long long ns) { g_timeout_ns.store(ns ? ns : 1ull); }

int mea_device_error(int* code, int clear) {
  if (!code) return MEA_ERR_NULL;
  if (cudaDeviceSynchronize() != cudaSuccess) return MEA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, mea::g_mea_error, sizeof(v)) != cudaSuccess) return MEA_ERR_CUDA;
  *code = static_cast<int>(v);
  if (clear) {
    unsigned int z = 0;
    if (cudaMemcpyToSymbol(mea::g_mea_error, &z, sizeof(z)) != cudaSuccess) return MEA_ERR_CUDA;
  }
  return MEA_OK;
}


int mea_wait_selftest(unsigned long long timeout_ns, int arrive, void* stream) {
  const unsigned long long t = timeout_ns ? timeout_ns : g_timeout_ns.load();
  clear_stale_launch_error();
  mea::mea_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(t, arrive);
  return cudaGetLastError() == cudaSuccess ? MEA_OK : MEA_ERR_CUDA;
}

size_t mea_backward_workspace_size(int total_q, int n_heads_q) {
  if (total_q < 0 || n_heads_q < 1) return 0;
  return 2 * (static_cast<size_t>(total_q) + 128) * static_cast<size_t>(n_heads_q) *
             sizeof(float) + mea::kBwdOrderMax * sizeof(int) + 256;
}

int mea_backward(const void* q, const void* k, const void* v, const void* out, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q,
                 const int32_t* cu_seqlens_k, int n_seqs, int total_q, int total_k,
                 int max_seqlen_q, int max_seqlen_k, int n_heads_q, int n_heads_kv, int head_dim,
                 float scale, int mask_kind, const float* alibi_slopes, int dtype, void* workspace,
                 size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !cu_seqlens_q ||
      !cu_seqlens_k)
    return MEA_ERR_NULL;
  if (n_seqs < 1 || n_seqs > 65535 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 ||
      max_seqlen_k < 0 || max_seqlen_q > total_q || max_seqlen_k > total_k)
    return MEA_ERR_SHAPE;
  if (n_heads_q < 1 || n_heads_kv < 1 || n_heads_q % n_heads_kv != 0) return MEA_ERR_HEADS;
  if (!dec_head_dim_ok(head_dim) || head_dim > 128) return MEA_ERR_HEAD_DIM;
  if (dtype != MEA_F16 && dtype != MEA_BF16) return MEA_ERR_DTYPE;
  if (mask_kind != MEA_MASK_NONE && mask_kind != MEA_MASK_CAUSAL) return MEA_ERR_MASK;
  if (!std::isfinite(scale)) return MEA_ERR_SCALE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4) || !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4) ||
      (alibi_slopes && !aligned(alibi_slopes, 4)))
    return MEA_ERR_ALIGN;
  if (!workspace || !aligned(workspace, 16) ||
      workspace_bytes < mea_backward_workspace_size(total_q, n_heads_q))
    return MEA_ERR_WORKSPACE;
  DeviceInfo di;
  if (int rc = current_device_info(di); rc != MEA_OK) return rc;
  if (total_q == 0 && total_k == 0) return MEA_OK;

  mea::BwdParams p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.out = out;
  p.lse = lse;
  p.dout = dout;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.t_pad = total_q + 128;
  p.nd = static_cast<float*>(workspace);
  p.na = p.nd + static_cast<size_t>(p.t_pad) * n_heads_q;
  p.lin_bias = (alibi_slopes != nullptr && mask_kind == MEA_MASK_CAUSAL) ? 1 : 0;
  p.order = n_seqs <= mea::kBwdOrderMax
                ? reinterpret_cast<int*>(p.na + static_cast<size_t>(p.t_pad) * n_heads_q)
                : nullptr;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.slopes = alibi_slopes;
  p.n_seqs = n_seqs;
  p.total_q = total_q;
  p.total_k = total_k;
  p.hq = n_heads_q;
  p.hkv = n_heads_kv;
  p.dh = head_dim;
  p.R = n_heads_q / n_heads_kv;
  // dQ: one CTA runs the same query tile for mq heads in turn (of one KV group when R allows)
  p.mq = n_heads_q % 4 == 0 ? 4 : (n_heads_q % 2 == 0 ? 2 : 1);
  const uint64_t dq_ctas =
      static_cast<uint64_t>(n_heads_q / p.mq) * ((static_cast<uint64_t>(max_seqlen_q) + 127) / 128);
  if (dq_ctas > 0x7fffffffull) return MEA_ERR_SHAPE;  // the dQ grid's x dimension
  p.scale = scale;
  p.c1 = scale * 1.4426950408889634f;
  BwdMaps m;
  const uint64_t tq_rows = total_q > 0 ? static_cast<uint64_t>(total_q) : 1;
  const uint64_t tk_rows = total_k > 0 ? static_cast<uint64_t>(total_k) : 1;
  if (!encode_3d(&m.q, q, dtype, head_dim, n_heads_q, tq_rows, 64, 1, 128) ||
      !encode_3d(&m.dout, dout, dtype, head_dim, n_heads_q, tq_rows, 64, 1, 128) ||
      !encode_3d(&m.k, k, dtype, head_dim, n_heads_kv, tk_rows, 64, 1, 128) ||
      !encode_3d(&m.v, v, dtype, head_dim, n_heads_kv, tk_rows, 64, 1, 128))
    return MEA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool causal = mask_kind == MEA_MASK_CAUSAL;
  const bool alibi = alibi_slopes != nullptr;
  if (head_dim > 64)
    return dtype == MEA_BF16
               ? launch_bwd_d<128, true>(causal, alibi, m, p, max_seqlen_q, max_seqlen_k, s)
               : launch_bwd_d<128, false>(causal, alibi, m, p, max_seqlen_q, max_seqlen_k, s);
  return dtype == MEA_BF16
             ? launch_bwd_d<64, true>(causal, alibi, m, p, max_seqlen_q, max_seqlen_k, s)
             : launch_bwd_d<64, false>(causal, alibi, m, p, max_seqlen_q, max_seqlen_k, s);
}

int mea_forward(const void* q, const void* k, const void* v, void* out, float* lse,
                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int n_seqs,
                int total_q, int total_k, int max_seqlen_q, int n_heads_q, int n_heads_kv,
                int head_dim, float scale, int mask_kind, const float* alibi_slopes, int dtype,
                void* stream) {
  return forward_impl(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, n_seqs, total_q, total_k,
                      max_seqlen_q, n_heads_q, n_heads_kv, head_dim, scale, mask_kind,
                      alibi_slopes, dtype, false, 1.f, 1.f, stream);
}

int mea_forward_fp8(const void* q, const void* k, const void* v, void* out, float* lse,
                    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int n_seqs,
                    int total_q, int total_k, int max_seqlen_q, int n_heads_q, int n_heads_kv,
                    int head_dim, float scale, int mask_kind, const float* alibi_slopes,
                    float q_descale, float k_descale, float v_descale, int out_dtype,
                    void* stream) {
  return forward_impl(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, n_seqs, total_q, total_k,
                      max_seqlen_q, n_heads_q, n_heads_kv, head_dim, scale, mask_kind,
                      alibi_slopes, out_dtype, true, q_descale * k_descale, v_descale, stream);
}

size_t mea_decode_workspace_size(int n_seqs, int total_k, int n_heads_q, int n_heads_kv,
                                 int head_dim, int split_keys) {
  DeviceInfo di;
  int sms = (current_device_info(di) == MEA_OK) ? di.sms : 148;
  DecLayout L;
  if (!dec_layout(n_seqs, total_k, n_heads_q, n_heads_kv, head_dim, split_keys, sms, L)) return 0;
  return L.total;
}

int mea_decode_splitkv(const void* q, const void* k, const void* v, void* out, float* lse,
                       const int32_t* cu_seqlens_k, int n_seqs, int total_k, int max_seqlen_k,
                       int n_heads_q, int n_heads_kv, int head_dim, float scale, int mask_kind,
                       const float* alibi_slopes, int dtype, void* workspace,
                       size_t workspace_bytes, int split_keys, void* stream) {
  if (!q || !k || !v || !out || !cu_seqlens_k) return MEA_ERR_NULL;
  if (n_seqs < 1 || total_k < 0 || max_seqlen_k < 0 || max_seqlen_k > total_k)
    return MEA_ERR_SHAPE;
  if (split_keys < 0 || split_keys % 64) return MEA_ERR_SHAPE;
  if (n_heads_q < 1 || n_heads_kv < 1 || n_heads_q % n_heads_kv != 0) return MEA_ERR_HEADS;
  if (!dec_head_dim_ok(head_dim)) return MEA_ERR_HEAD_DIM;
  if (dtype != MEA_F16 && dtype != MEA_BF16) return MEA_ERR_DTYPE;
  if (mask_kind != MEA_MASK_NONE && mask_kind != MEA_MASK_CAUSAL) return MEA_ERR_MASK;
  if (!std::isfinite(scale)) return MEA_ERR_SCALE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      (lse && !aligned(lse, 4)) || !aligned(cu_seqlens_k, 4) ||
      (alibi_slopes && !aligned(alibi_slopes, 4)))
    return MEA_ERR_ALIGN;
  if (!workspace || !aligned(workspace, 256)) return MEA_ERR_WORKSPACE;
  // The automatic chunk size depends on the SM count; an explicit one does not, so a
  // too-small workspace is reported before the device is queried.
  DeviceInfo di;
  int dev_rc = MEA_OK;
  if (split_keys == 0 && (dev_rc = current_device_info(di)) != MEA_OK) return dev_rc;
  DecLayout L;
  if (!dec_layout(n_seqs, total_k, n_heads_q, n_heads_kv, head_dim, split_keys,
                  split_keys == 0 ? di.sms : 0, L))
    return MEA_ERR_SHAPE;
  if (workspace_bytes < L.total) return MEA_ERR_WORKSPACE;
  if (split_keys != 0 && (dev_rc = current_device_info(di)) != MEA_OK) return dev_rc;

  const int R = n_heads_q / n_heads_kv;
  mea::DecParams p{};
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.cu_k = cu_seqlens_k;
  p.slopes = alibi_slopes;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.lse_off);
  p.n_seqs = n_seqs;
  p.hq = n_heads_q;
  p.dh = head_dim;
  p.R = R;
  p.RB = decode_rb(R);
  p.n_hb = n_heads_q / p.RB;
  p.chunk = L.chunk;
  p.n_slots = L.n_slots;
  p.n_items = static_cast<long long>(L.n_slots) * p.n_hb;
  p.c1 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();

  CUtensorMap tk, tv;
  const uint64_t tk_rows = total_k > 0 ? static_cast<uint64_t>(total_k) : 1;
  if (!encode_3d(&tk, k, dtype, head_dim, n_heads_kv, tk_rows, 64, 1, 64) ||
      !encode_3d(&tv, v, dtype, head_dim, n_heads_kv, tk_rows, 64, 1, 64))
    return MEA_ERR_CUDA;
  const int grid = total_k > 0 ? static_cast<int>(p.n_items < di.sms ? p.n_items : di.sms) : 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool alibi = alibi_slopes != nullptr;
  if (head_dim > 128)
    return dtype == MEA_BF16 ? launch_dec_d<256, true>(alibi, tk, tv, p, grid, n_heads_kv, s)
                             : launch_dec_d<256, false>(alibi, tk, tv, p, grid, n_heads_kv, s);
  if (head_dim > 64)
    return dtype == MEA_BF16 ? launch_dec_d<128, true>(alibi, tk, tv, p, grid, n_heads_kv, s)
                             : launch_dec_d<128, false>(alibi, tk, tv, p, grid, n_heads_kv, s);
  return dtype == MEA_BF16 ? launch_dec_d<64, true>(alibi, tk, tv, p, grid, n_heads_kv, s)
                           : launch_dec_d<64, false>(alibi, tk, tv, p, grid, n_heads_kv, s);
}

int mea_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* block_table, const int32_t* cu_seqlens_k, void* out,
                     float* lse, int n_seqs, int num_blocks, int block_size, int max_blocks,
                     int total_k, int max_seqlen_k, int n_heads_q, int n_heads_kv, int head_dim,
                     float scale, int mask_kind, const float* alibi_slopes, int dtype,
                     void* workspace, size_t workspace_bytes, int split_keys, void* stream) {
  if (!q || !k_cache || !v_cache || !block_table || !cu_seqlens_k || !out) return MEA_ERR_NULL;
  if (n_seqs < 1 || num_blocks < 1 || max_blocks < 1 || total_k < 0 || max_seqlen_k < 0 ||
      max_seqlen_k > total_k || static_cast<long long>(max_blocks) * block_size < max_seqlen_k)
    return MEA_ERR_SHAPE;
  if (!(block_size == 16 || block_size == 32 || (block_size >= 64 && block_size % 64 == 0)))
    return MEA_ERR_SHAPE;
  if (split_keys < 0 || split_keys % 64) return MEA_ERR_SHAPE;
  if (n_heads_q < 1 || n_heads_kv < 1 || n_heads_q % n_heads_kv != 0) return MEA_ERR_HEADS;
  if (!dec_head_dim_ok(head_dim)) return MEA_ERR_HEAD_DIM;
  if (dtype != MEA_F16 && dtype != MEA_BF16) return MEA_ERR_DTYPE;
  if (mask_kind != MEA_MASK_NONE && mask_kind != MEA_MASK_CAUSAL) return MEA_ERR_MASK;
  if (!std::isfinite(scale)) return MEA_ERR_SCALE;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      (lse && !aligned(lse, 4)) || !aligned(cu_seqlens_k, 4) || !aligned(block_table, 4) ||
      (alibi_slopes && !aligned(alibi_slopes, 4)))
    return MEA_ERR_ALIGN;
  if (!workspace || !aligned(workspace, 256)) return MEA_ERR_WORKSPACE;
  DeviceInfo di;
  int dev_rc = MEA_OK;
  if (split_keys == 0 && (dev_rc = current_device_info(di)) != MEA_OK) return dev_rc;
  DecLayout L;
  if (!dec_layout(n_seqs, total_k, n_heads_q, n_heads_kv, head_dim, split_keys,
                  split_keys == 0 ? di.sms : 0, L))
    return MEA_ERR_SHAPE;
  if (workspace_bytes < L.total) return MEA_ERR_WORKSPACE;
  if (split_keys != 0 && (dev_rc = current_device_info(di)) != MEA_OK) return dev_rc;

  const int R = n_heads_q / n_heads_kv;
  mea::DecParams p{};
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.cu_k = cu_seqlens_k;
  p.slopes = alibi_slopes;
  p.block_table = block_table;
  p.block_size = block_size;
  p.max_blocks = max_blocks;
  p.num_blocks = num_blocks;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.lse_off);
  p.n_seqs = n_seqs;
  p.hq = n_heads_q;
  p.dh = head_dim;
  p.R = R;
  p.RB = decode_rb(R);
  p.n_hb = n_heads_q / p.RB;
  p.chunk = L.chunk;
  p.n_slots = L.n_slots;
  p.n_items = static_cast<long long>(L.n_slots) * p.n_hb;
  p.c1 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();

  CUtensorMap tk, tv;
  const uint32_t rows = block_size < 64 ? static_cast<uint32_t>(block_size) : 64u;
  // Head dims equal to the kernel's width (64, 128, 256) take one box per block (every atom at
  // once); the others one box per atom, whose zero fill covers the columns past head_dim.
  p.box5 = (head_dim == 64 || head_dim == 128 || head_dim == 256) ? 1 : 0;
  p.lay_log2 = p.box5 ? (rows == 16 ? 4 : rows == 32 ? 5 : 6) : 6;
  if (p.box5) {
    if (!encode_paged5(&tk, k_cache, dtype, head_dim, n_heads_kv, block_size, num_blocks, rows) ||
        !encode_paged5(&tv, v_cache, dtype, head_dim, n_heads_kv, block_size, num_blocks, rows))
      return MEA_ERR_CUDA;
  } else if (!encode_4d(&tk, k_cache, dtype, head_dim, n_heads_kv, block_size, num_blocks, 64, 1,
                        rows, 1) ||
             !encode_4d(&tv, v_cache, dtype, head_dim, n_heads_kv, block_size, num_blocks, 64, 1,
                        rows, 1)) {
    return MEA_ERR_CUDA;
  }
  const int grid = total_k > 0 ? static_cast<int>(p.n_items < di.sms ? p.n_items : di.sms) : 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool alibi = alibi_slopes != nullptr;
  if (head_dim > 128)
    return dtype == MEA_BF16
               ? launch_dec_d<256, true, true>(alibi, tk, tv, p, grid, n_heads_kv, s)
               : launch_dec_d<256, false, true>(alibi, tk, tv, p, grid, n_heads_kv, s);
  if (head_dim > 64)
    return dtype == MEA_BF16
               ? launch_dec_d<128, true, true>(alibi, tk, tv, p, grid, n_heads_kv, s)
               : launch_dec_d<128, false, true>(alibi, tk, tv, p, grid, n_heads_kv, s);
  return dtype == MEA_BF16 ? launch_dec_d<64, true, true>(alibi, tk, tv, p, grid, n_heads_kv, s)
                           : launch_dec_d<64, false, true>(alibi, tk, tv, p, grid, n_heads_kv, s);
}

int mea_decode_splitkv_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                               const int32_t* cu_seqlens_k, int n_seqs, int total_k,
                               int max_seqlen_k, int n_heads_q, int n_heads_kv, int head_dim,
                               float scale, int mask_kind, const float* alibi_slopes, int dtype,
                               int split_keys, void* stream) {
  if (!q || !k || !v || !out || !cu_seqlens_k) return MEA_ERR_NULL;
  if (n_seqs < 1 || total_k < 0 || max_seqlen_k < 0 || max_seqlen_k > total_k)
    return MEA_ERR_SHAPE;
  if (split_keys < 0 || split_keys % 64) return MEA_ERR_SHAPE;
  if (n_heads_q < 1 || n_heads_kv < 1 || n_heads_q % n_heads_kv != 0) return MEA_ERR_HEADS;
  if (!dec_head_dim_ok(head_dim)) return MEA_ERR_HEAD_DIM;
  if (dtype != MEA_F16 && dtype != MEA_BF16) return MEA_ERR_DTYPE;
  if (mask_kind != MEA_MASK_NONE && mask_kind != MEA_MASK_CAUSAL) return MEA_ERR_MASK;
  if (!std::isfinite(scale)) return MEA_ERR_SCALE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      (lse && !aligned(lse, 4)) || !aligned(cu_seqlens_k, 4) ||
      (alibi_slopes && !aligned(alibi_slopes, 4)))
    return MEA_ERR_ALIGN;

  // Chunk size: as given, or the library's choice doubled until the partials fit the array.
  const size_t limit = MEA_DECODE_NOALLOC_SCRATCH_BYTES;
  DecLayout L;
  DeviceInfo di;
  if (split_keys != 0) {
    if (!dec_layout(n_seqs, total_k, n_heads_q, n_heads_kv, head_dim, split_keys, 0, L))
      return MEA_ERR_SHAPE;
    if (L.total > limit) return MEA_ERR_SCRATCH_LIMIT;
    if (int rc = current_device_info(di); rc != MEA_OK) return rc;
  } else {
    if (int rc = current_device_info(di); rc != MEA_OK) return rc;
    if (!dec_layout(n_seqs, total_k, n_heads_q, n_heads_kv, head_dim, 0, di.sms, L))
      return MEA_ERR_SHAPE;
    int chunk = L.chunk;
    while (L.total > limit && chunk < (1 << 24) && chunk < total_k) {
      chunk *= 2;
      if (!dec_layout(n_seqs, total_k, n_heads_q, n_heads_kv, head_dim, chunk, 0, L))
        return MEA_ERR_SHAPE;
    }
    if (L.total > limit) return MEA_ERR_SCRATCH_LIMIT;
  }
  void* scratch = nullptr;
  if (int rc = noalloc_scratch_address(&scratch); rc != MEA_OK) return rc;

  const int R = n_heads_q / n_heads_kv;
  mea::DecParams p{};
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.cu_k = cu_seqlens_k;
  p.slopes = alibi_slopes;
  p.ws_o = static_cast<float*>(scratch);
  p.ws_lse = reinterpret_cast<float*>(static_cast<char*>(scratch) + L.lse_off);
  p.n_seqs = n_seqs;
  p.hq = n_heads_q;
  p.dh = head_dim;
  p.R = R;
  p.RB = decode_rb(R);
  p.n_hb = n_heads_q / p.RB;
  p.chunk = L.chunk;
  p.n_slots = L.n_slots;
  p.n_items = static_cast<long long>(L.n_slots) * p.n_hb;
  p.c1 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load();

  CUtensorMap tk, tv;
  const uint64_t tk_rows = total_k > 0 ? static_cast<uint64_t>(total_k) : 1;
  if (!encode_3d(&tk, k, dtype, head_dim, n_heads_kv, tk_rows, 64, 1, 64) ||
      !encode_3d(&tv, v, dtype, head_dim, n_heads_kv, tk_rows, 64, 1, 64))
    return MEA_ERR_CUDA;
  const int grid = total_k > 0 ? static_cast<int>(p.n_items < di.sms ? p.n_items : di.sms) : 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool alibi = alibi_slopes != nullptr;
  if (head_dim > 128)
    return dtype == MEA_BF16 ? launch_dec_d<256, true>(alibi, tk, tv, p, grid, n_heads_kv, s)
                             : launch_dec_d<256, false>(alibi, tk, tv, p, grid, n_heads_kv, s);
  if (head_dim > 64)
    return dtype == MEA_BF16 ? launch_dec_d<128, true>(alibi, tk, tv, p, grid, n_heads_kv, s)
                             : launch_dec_d<128, false>(alibi, tk, tv, p, grid, n_heads_kv, s);
  return dtype == MEA_BF16 ? launch_dec_d<64, true>(alibi, tk, tv, p, grid, n_heads_kv, s)
                           : launch_dec_d<64, false>(alibi, tk, tv, p, grid, n_heads_kv, s);
}

}  // extern "C"
