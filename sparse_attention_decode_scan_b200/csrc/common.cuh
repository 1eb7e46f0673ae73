// Shared device helpers of liblsa: element loads, status word, cache addressing.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa.h"

namespace lsa {

// Workspace layout: [0, 256) status word area, then per-op regions (host side
// computes offsets; see abi.cu).
constexpr size_t kStatusBytes = 256;

struct DevStatus {
  int32_t code;      // first recorded lsa_status (0 = none)
  int32_t detail0;   // e.g. offending row
  int32_t detail1;   // e.g. offending block id / position
  int32_t count;     // number of recorded errors
};

// Kept out of line: it is on error paths only, and inlining its atomics at
// every call site would grow the kernels' code (cold code is fetched from
// memory at each launch).
static __device__ __noinline__ void record_error(DevStatus* st, int code, int d0, int d1) {
  if (st == nullptr) return;
  if (atomicCAS(&st->code, 0, code) == 0) {
    st->detail0 = d0;
    st->detail1 = d1;
  }
  atomicAdd(&st->count, 1);
}

// Unsigned division by an invariant d >= 1 as a multiply-high, an add and a
// shift (Granlund and Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994, the round-up multiplier m' = floor(2^(32+l)/d)+1
// with l = ceil(log2 d), stored as m' - 2^32); exact for n < 2^31.
struct DivU32 {
  uint32_t d, m;
  int l;
};

__host__ __device__ inline DivU32 make_divu32(uint32_t d) {
  DivU32 v;
  v.d = d;
  int l = 0;
  while ((1ull << l) < d) ++l;
  v.l = l;
  v.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << l) - d)) / d + 1);
  return v;
}

__device__ __forceinline__ uint32_t divu32(const DivU32& v, uint32_t n) { return (__umulhi(n, v.m) + n) >> v.l; }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float e4m3_to_float(uint8_t b) {
  __nv_fp8_e4m3 v;
  v.__x = b;
  return static_cast<float>(v);
}

template <int DT>
__device__ __forceinline__ float load_elem(const void* p, int64_t i);

template <>
__device__ __forceinline__ float load_elem<LSA_F32>(const void* p, int64_t i) {
  return __ldg(reinterpret_cast<const float*>(p) + i);
}
template <>
__device__ __forceinline__ float load_elem<LSA_BF16>(const void* p, int64_t i) {
  return bf16_bits_to_float(__ldg(reinterpret_cast<const unsigned short*>(p) + i));
}
template <>
__device__ __forceinline__ float load_elem<LSA_FP8_E4M3>(const void* p, int64_t i) {
  return e4m3_to_float(reinterpret_cast<const uint8_t*>(p)[i]);
}

// Loads 8 consecutive elements starting at element i (i multiple of 8) as floats.
template <int DT>
__device__ __forceinline__ void load8(const void* p, int64_t i, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<LSA_F32>(const void* p, int64_t i, float (&v)[8]) {
  const float4* q = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
  float4 a = __ldg(q), b = __ldg(q + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<LSA_BF16>(const void* p, int64_t i, float (&v)[8]) {
  uint4 a = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned short*>(p) + i));
  uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = __uint_as_float(w[j] << 16);
    v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
  }
}
template <>
__device__ __forceinline__ void load8<LSA_FP8_E4M3>(const void* p, int64_t i, float (&v)[8]) {
  uint2 a = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(p) + i));
  uint32_t w[2] = {a.x, a.y};
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = e4m3_to_float(static_cast<uint8_t>(w[j >> 2] >> (8 * (j & 3))));
}

// Flat stored row of logical position `pos` of sequence `b`, or -1 if the
// block-table entry is outside [0, n_blocks).
struct CacheAddr {
  const int32_t* block_table;
  int32_t max_blocks;
  int32_t block_size;  // 0 = contiguous
  int64_t n_blocks;
  int64_t max_len;

  __device__ __forceinline__ int64_t row(int b, int64_t pos) const {
    if (block_size == 0) return static_cast<int64_t>(b) * max_len + pos;
    int64_t lb = pos / block_size;
    if (lb >= max_blocks) return -1;
    int32_t blk = __ldg(block_table + static_cast<int64_t>(b) * max_blocks + lb);
    if (blk < 0 || blk >= n_blocks) return -1;
    return static_cast<int64_t>(blk) * block_size + (pos - lb * block_size);
  }
};

// Order-preserving 32-bit key of a score (larger score -> larger key).  -0.0
// maps like +0.0; -inf and NaN map to 0, the key that is never selected.
__device__ __forceinline__ uint32_t order_key(float f) {
  if (!(f == f) || f == -INFINITY) return 0u;
  uint32_t u = __float_as_uint(f);
  if (f == 0.f) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Bins of the first top-k digit (key bits [31:20]).
constexpr int kTopkBins1 = 4096;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace lsa
