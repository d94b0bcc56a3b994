// Memory injection of the linear (DGA) layers: each query's initial state S_ext
// is the sum of its selected documents' recurrent states
// ("MSA x Qwen3.5" model card, "Architecture summary": the top-k documents'
// recurrent states are summed into S_ext, the initial state of the query
// path's gated delta rule).
//
// A pure HBM stream: every selected state is read once per query and one fp32
// state is written.  Each thread owns one 16-byte vector of the state and keeps
// up to eight of the query's selected documents' vectors in flight before
// adding them, in rank order, in fp32.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 8;  // loads in flight per thread

template <typename T>
__global__ void __launch_bounds__(kThreads) state_sum_kernel(const T* __restrict__ states, int64_t D, int64_t S,
                                                             const int32_t* __restrict__ idx, int k,
                                                             float* __restrict__ out, int32_t* err_flag) {
  constexpr int VN = Vec<T>::N;  // elements per 16-byte vector
  const int64_t nv = S / VN;
  const int64_t b = blockIdx.y;
  const int64_t v = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (v >= nv) return;
  const int32_t* row = idx + b * k;
  float acc[VN];
#pragma unroll
  for (int i = 0; i < VN; ++i) acc[i] = 0.f;
  for (int r0 = 0; r0 < k; r0 += kBatch) {
    uint4 u[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int r = r0 + q;
      const int64_t j = r < k ? (int64_t)__ldg(row + r) : 0;
      const bool ok = r < k && j >= 0 && j < D;
      if (r < k && !ok && v == 0) raise_flag(err_flag, MSA_FLAG_INDEX_OOB);
      u[q] = ok ? __ldg(reinterpret_cast<const uint4*>(states + j * S) + v) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      float x[VN];
      unpack(u[q], x);
#pragma unroll
      for (int i = 0; i < VN; ++i) acc[i] += x[i];
    }
  }
  float4* o = reinterpret_cast<float4*>(out + b * S + v * VN);
#pragma unroll
  for (int i = 0; i < VN; i += 4) o[i / 4] = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
}

template <typename T>
cudaError_t state_sum_t(const void* states, int64_t D, int64_t S, const int32_t* idx, int64_t B, int k,
                        float* out, int32_t* err_flag, cudaStream_t s) {
  const int64_t nv = S / Vec<T>::N;
  const int64_t gx = (nv + kThreads - 1) / kThreads;
  if (gx > 0x7fffffffLL) return cudaErrorInvalidValue;
  count_launch();
  state_sum_kernel<T><<<dim3((unsigned)gx, (unsigned)B), kThreads, 0, s>>>(
      reinterpret_cast<const T*>(states), D, S, idx, k, out, err_flag);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_sum(msa_dtype dt, const void* states, int64_t D, int64_t S, const int32_t* idx,
                             int64_t B, int k, float* out, int32_t* err_flag, cudaStream_t s) {
  return dt == MSA_F32 ? state_sum_t<float>(states, D, S, idx, B, k, out, err_flag, s)
                       : state_sum_t<__nv_bfloat16>(states, D, S, idx, B, k, out, err_flag, s);
}

}  // namespace msa
