// Shared device helpers of the MSA memory-path library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "msa.h"

namespace msa {

// ---------------------------------------------------------------- storage types
template <typename T> struct Vec;  // one 16-byte vector of T
template <> struct Vec<float> {
  static constexpr int N = 4;
};
template <> struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
};

__device__ __forceinline__ void unpack(const uint4& u, float (&f)[4]) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void unpack(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);          // bf16 -> fp32 is exact
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ uint4 pack(const float (&f)[4]) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint4 pack(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// ---------------------------------------------------------------- ordered keys
// A float's bits mapped to an unsigned integer with the same order (for
// atomicMax and radix/bitonic selection).  Key 0 is below every float and is
// read back as -inf ("no chunk seen").
__device__ __forceinline__ uint32_t float_to_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
  if (k == 0u) return __uint_as_float(0xff800000u);  // -inf
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

__device__ __forceinline__ void raise_flag(int32_t* flag, int bits) {
  if (flag) atomicOr(flag, bits);
}

// Index of the document owning chunk c: the j with off[j] <= c < off[j+1]
// (largest j with off[j] <= c); off is non-decreasing, length D+1.
// Programmatic dependent launch: wait for the previous kernel on the stream to
// finish (and its writes to be visible); let the next kernel start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ int64_t owner_doc(const int64_t* __restrict__ off, int64_t D, int64_t c) {
  int64_t lo = 0, hi = D;  // answer in [lo, hi)
  while (hi - lo > 1) {
    int64_t mid = (lo + hi) >> 1;
    if (__ldg(off + mid) <= c) lo = mid; else hi = mid;
  }
  return lo;
}

// owner_doc for a whole warp at once, with 32-way probes: every round each lane
// tests one of 32 evenly spaced offsets and a ballot keeps the last range that
// can still hold c, so ~log32(D) dependent loads instead of log2(D).  All 32
// lanes must call it with the same c; all get the same answer.  Requires
// off[0] <= c.
__device__ __forceinline__ int64_t warp_owner_doc(const int64_t* __restrict__ off, int64_t D, int64_t c,
                                                  int lane) {
  int64_t lo = 0, hi = D;  // answer in [lo, hi), off[lo] <= c
  while (hi - lo > 1) {
    const int64_t step = (hi - lo + 31) / 32;
    const int64_t pos = lo + (int64_t)lane * step;
    const bool le = pos < hi && __ldg(off + pos) <= c;
    const unsigned m = __ballot_sync(0xffffffffu, le);
    const int last = 31 - __clz(m);
    lo += (int64_t)last * step;
    hi = min(hi, lo + step);
  }
  return lo;
}

// warp_owner_doc that first looks at the 32 documents around the proportional
// guess c * D / C (one coalesced load; right whenever the documents' chunk
// counts are close to uniform) and searches only if the owner is not among
// them.  All 32 lanes must call it with the same c; all get the same answer,
// a document in [0, D) whatever the offsets hold.
__device__ __forceinline__ int64_t warp_owner_doc_near(const int64_t* __restrict__ off, int64_t D, int64_t C,
                                                       int64_t c, int lane) {
  // a guess only (a miss falls back to the full search): fp32 keeps it within a
  // document for D up to ~2^24, without a double-precision division
  int64_t g = (C > 0 ? (int64_t)((float)c * ((float)D / (float)C)) : 0) - 16;
  if (g > D - 32) g = D - 32;
  if (g < 0) g = 0;
  const int64_t j = g + lane;
  const unsigned m = __ballot_sync(0xffffffffu, j < D && __ldg(off + j) <= c);
  if (m != 0) {
    const int last = 31 - __clz(m);
    // the window's next document starts after c (or there is none): it is the owner
    if (last < 31 || g + 32 >= D) return g + last;
  }
  return warp_owner_doc(off, D, c, lane);
}

// Owning document of chunk c0 + lane for the 32 consecutive chunks of a warp
// (-1 for chunks >= C).  One warp-wide search for c0, then each lane counts the
// document boundaries at or below its chunk among the next 32 (documents with no
// chunks are boundaries too) by a binary search over the lanes' boundaries,
// which valid offsets leave sorted (invalid ones give some count in [0, 32],
// never an index outside the window); falls back to a per-lane search when 32
// boundaries do not cover the warp's chunks.  All 32 lanes must call it.
__device__ __forceinline__ int warp_chunk_docs(const int64_t* __restrict__ off, int64_t D, int64_t C, int64_t c0,
                                               int lane) {
  if (c0 >= C) return -1;
  const int64_t j0 = warp_owner_doc_near(off, D, C, c0, lane);
  const int64_t c = c0 + lane;
  const int64_t bidx = j0 + 1 + lane;
  const int64_t b = __ldg(off + (bidx < D ? bidx : D));
  // boundary l relative to c0, clamped to [0, 32]: a 32-bit sorted list
  const int64_t rb = b - c0;
  const int r = rb < 0 ? 0 : (rb > 32 ? 32 : (int)rb);
  int cnt = 0;  // boundaries r_l <= lane
#pragma unroll
  for (int step = 16; step > 0; step >>= 1)
    if (__shfl_sync(0xffffffffu, r, cnt + step - 1) <= lane) cnt += step;
  if (__shfl_sync(0xffffffffu, r, cnt & 31) <= lane && cnt == 31) cnt = 32;
  const int64_t b31 = __shfl_sync(0xffffffffu, b, 31);
  const bool covered = b31 > c0 + 31 || j0 + 32 >= D;
  if (c >= C) return -1;
  if (covered) return (int)(j0 + cnt);
  return (int)owner_doc(off, D, c);
}

}  // namespace msa
