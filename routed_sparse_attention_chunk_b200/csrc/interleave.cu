// Memory Interleave ("MSA: Memory Sparse Attention" README, Figure 3 caption:
// an optional multi-round interleave for multi-hop questions; FAQ "What is
// Memory Interleave?": several rounds of routing that jump across scattered
// memory segments).  Each round routes, selects k documents not selected in an
// earlier round, and attends over every round's documents so far; the next
// round's router query is the caller's linear map of this round's attention
// output.  This file holds that map's kernel and the entry point that runs the
// rounds from the library's kernels.
//
// The map is a small dense product (rows = B * Tq query tokens, K = Hq * d,
// N = Hr * dr): a CUDA-core tiled kernel with fp32 accumulation, one CTA per
// BM x 64 output tile, operands staged through shared memory in steps of 32.
// With few rows (64 query tokens) that is 64 CTAs, each walking all of K in
// dependent steps, so the map is latency-bound: a few hundred microseconds for
// K = 4096, N = 1024, against the routing scan's ~0.5 ms on a 100M-token bank.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "msa.h"

namespace msa {
namespace {

constexpr int kBN = 64, kBK = 32, kThreads = 256;

template <typename T, int BM>
__global__ void __launch_bounds__(kThreads) project_kernel(const T* __restrict__ A, const T* __restrict__ W,
                                                           T* __restrict__ out, int64_t rows, int K, int N) {
  constexpr int TM = BM / 16;  // rows per thread; 16 x 16 threads each own TM x 4 outputs
  __shared__ float As[kBK][BM + 4];
  __shared__ float Ws[kBK][kBN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t r0 = (int64_t)blockIdx.y * BM;
  const int c0 = blockIdx.x * kBN;
  float acc[TM][4];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += kBK) {
    for (int i = threadIdx.x; i < BM * kBK; i += kThreads) {
      const int rr = i / kBK, kk = i % kBK;
      const int64_t row = r0 + rr;
      const int kc = k0 + kk;
      As[kk][rr] = (row < rows && kc < K) ? to_f32(A[row * K + kc]) : 0.f;
    }
    for (int i = threadIdx.x; i < kBK * kBN; i += kThreads) {
      const int kk = i / kBN, cc = i % kBN;
      const int kc = k0 + kk, col = c0 + cc;
      Ws[kk][cc] = (kc < K && col < N) ? to_f32(W[(int64_t)kc * N + col]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kBK; ++kk) {
      float a[TM], w[4];
#pragma unroll
      for (int i = 0; i < TM; ++i) a[i] = As[kk][ty * TM + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = Ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int64_t row = r0 + ty * TM + i;
    if (row >= rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = c0 + tx * 4 + j;
      if (col < N) out[row * N + col] = from_f32<T>(acc[i][j]);
    }
  }
}

template <typename T>
cudaError_t project_t(const void* in, const void* W, void* out, int64_t rows, int K, int N, cudaStream_t s) {
  const T* a = static_cast<const T*>(in);
  const T* w = static_cast<const T*>(W);
  T* o = static_cast<T*>(out);
  const unsigned gx = (unsigned)((N + kBN - 1) / kBN);
  count_launch();
  if (rows >= 1024) {
    project_kernel<T, 64><<<dim3(gx, (unsigned)((rows + 63) / 64)), kThreads, 0, s>>>(a, w, o, rows, K, N);
  } else {
    project_kernel<T, 16><<<dim3(gx, (unsigned)((rows + 15) / 16)), kThreads, 0, s>>>(a, w, o, rows, K, N);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_project(msa_dtype dt, const void* in, const void* W, void* out, int64_t rows, int K, int N,
                           cudaStream_t s) {
  if (rows <= 0 || K <= 0 || N <= 0) return cudaSuccess;
  return dt == MSA_F32 ? project_t<float>(in, W, out, rows, K, N, s)
                       : project_t<__nv_bfloat16>(in, W, out, rows, K, N, s);
}

}  // namespace msa
