// Backward of step 2 for the selected documents: the gradient of their routing
// scores.  A document's score is the max over its chunks c and the query's
// tokens t of s(t, c) = (1/Hr) sum_h cos(Qr[t, h], K̄r[c, h]) ("MSA: Memory
// Sparse Attention" README, "Architecture"); the model card trains the router
// with an auxiliary routing loss it does not define, so the upstream gradient
// d_score of each selected document is an input.  The max passes it to its
// argmax pair (the first in (chunk, token) order on ties) and the cosine's
// derivative spreads it over that token's Qr and that chunk's K̄r:
//   dQr[t*, h] += g/Hr (k / (|q| |k|) - cos q / |q|^2)
//   dK̄r[c*, h] += g/Hr (q / (|q| |k|) - cos k / |k|^2)
// Two launches: route_bwd_scan_kernel, grid (splits, k, B), recomputes s for
// its share of the document's (chunk, token) pairs (one pair per thread, fp32)
// and leaves its best pair in the workspace; route_bwd_grad_kernel, grid
// (k, B), one warp per router head, picks the best pair over the splits and
// adds the gradient with fp32 atomics (a token or chunk shared by several
// documents or queries accumulates).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int kSplits = 16;
constexpr int kScanThreads = 256;

struct Cand {
  float s;
  int32_t pair;  // c_rel * Tq + t; -1: none
};

__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
  return a.pair >= 0 && (b.pair < 0 || a.s > b.s || (a.s == b.s && a.pair < b.pair));
}

template <typename T>
__global__ void __launch_bounds__(kScanThreads) route_bwd_scan_kernel(RouteBwdArgs a, Cand* __restrict__ ws) {
  const int split = blockIdx.x, r = blockIdx.y;
  const int64_t b = blockIdx.z;
  __shared__ Cand red[kScanThreads / 32];
  Cand best{-INFINITY, -1};
  const int32_t j = __ldg(a.topk_idx + b * a.k + r);
  int64_t cs = 0, n = 0;
  if (j >= 0 && (int64_t)j < a.D) {
    cs = __ldg(a.doc_chunk_off + j);
    const int64_t ce = __ldg(a.doc_chunk_off + j + 1);
    if (cs >= 0 && ce <= a.C && ce >= cs) n = ce - cs;
  }
  int64_t pairs = n * a.Tq;
  if (pairs > 0x7fffffffLL) {  // the pair index is int32: such a document is skipped
    if (split == 0 && threadIdx.x == 0) raise_flag(a.err_flag, MSA_FLAG_INDEX_OOB);
    pairs = 0;
  }
  const int64_t per = (pairs + kSplits - 1) / kSplits;
  const int64_t p0 = split * per, p1 = min(pairs, p0 + per);
  const T* Q = reinterpret_cast<const T*>(a.Qr);
  const T* K = reinterpret_cast<const T*>(a.Krbar);
  constexpr int VN = Vec<T>::N;
  for (int64_t p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
    const int64_t c = cs + p / a.Tq;
    const int t = (int)(p % a.Tq);
    float s = 0.f;
    for (int h = 0; h < a.Hr; ++h) {
      const uint4* qv = reinterpret_cast<const uint4*>(Q + ((b * a.Tq + t) * a.Hr + h) * (int64_t)a.dr);
      const uint4* kv = reinterpret_cast<const uint4*>(K + (c * a.Hr + h) * (int64_t)a.dr);
      float dot = 0.f, nq = 0.f;
      for (int v = 0; v < a.dr / VN; ++v) {
        float x[VN], y[VN];
        unpack(__ldg(qv + v), x);
        unpack(__ldg(kv + v), y);
#pragma unroll
        for (int i = 0; i < VN; ++i) {
          dot = fmaf(x[i], y[i], dot);
          nq = fmaf(x[i], x[i], nq);
        }
      }
      s += dot / fmaxf(sqrtf(nq), 1e-12f) * __ldg(a.kr_rnorm + c * a.Hr + h);
    }
    const Cand cand{s / (float)a.Hr, (int32_t)p};
    if (better(cand, best)) best = cand;
  }
  // block argmax (ties to the lower pair index)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Cand other{__shfl_xor_sync(0xffffffffu, best.s, o), __shfl_xor_sync(0xffffffffu, best.pair, o)};
    if (better(other, best)) best = other;
  }
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kScanThreads / 32; ++w)
      if (better(red[w], best)) best = red[w];
    ws[(b * a.k + r) * kSplits + split] = best;
  }
}

template <typename T>
__global__ void route_bwd_grad_kernel(RouteBwdArgs a, const Cand* __restrict__ ws) {
  const int r = blockIdx.x;
  const int64_t b = blockIdx.y;
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t j = __ldg(a.topk_idx + b * a.k + r);
  if (j < 0 || (int64_t)j >= a.D) {
    if (threadIdx.x == 0) raise_flag(a.err_flag, MSA_FLAG_INDEX_OOB);
    return;
  }
  const int64_t cs = __ldg(a.doc_chunk_off + j), ce = __ldg(a.doc_chunk_off + j + 1);
  if (cs < 0 || ce > a.C || ce < cs) {
    if (threadIdx.x == 0) raise_flag(a.err_flag, MSA_FLAG_INDEX_OOB);
    return;
  }
  Cand best{-INFINITY, -1};
  for (int sp = 0; sp < kSplits; ++sp) {
    const Cand c = ws[(b * a.k + r) * kSplits + sp];
    if (better(c, best)) best = c;
  }
  if (best.pair < 0 || h >= a.Hr) return;  // a document with no chunks
  const int64_t c = cs + best.pair / a.Tq;
  const int t = best.pair % a.Tq;
  const T* q = reinterpret_cast<const T*>(a.Qr) + ((b * a.Tq + t) * a.Hr + h) * (int64_t)a.dr;
  const T* k = reinterpret_cast<const T*>(a.Krbar) + (c * a.Hr + h) * (int64_t)a.dr;
  float dot = 0.f, nq2 = 0.f, nk2 = 0.f;
  for (int i = lane; i < a.dr; i += 32) {
    const float x = to_f32(q[i]), y = to_f32(k[i]);
    dot = fmaf(x, y, dot);
    nq2 = fmaf(x, x, nq2);
    nk2 = fmaf(y, y, nk2);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
    nq2 += __shfl_xor_sync(0xffffffffu, nq2, o);
    nk2 += __shfl_xor_sync(0xffffffffu, nk2, o);
  }
  const float nq = fmaxf(sqrtf(nq2), 1e-12f), nk = fmaxf(sqrtf(nk2), 1e-12f);
  const float cosv = dot / (nq * nk);
  const float w = __ldg(a.d_score + b * a.k + r) / (float)a.Hr;
  float* dq = a.dQr + ((b * a.Tq + t) * a.Hr + h) * (int64_t)a.dr;
  float* dk = a.dKrbar + (c * a.Hr + h) * (int64_t)a.dr;
  for (int i = lane; i < a.dr; i += 32) {
    const float x = to_f32(q[i]), y = to_f32(k[i]);
    atomicAdd(dq + i, w * (y / (nq * nk) - cosv * x / (nq * nq)));
    atomicAdd(dk + i, w * (x / (nq * nk) - cosv * y / (nk * nk)));
  }
}

template <typename T>
cudaError_t route_bwd_t(const RouteBwdArgs& a, cudaStream_t s) {
  Cand* ws = static_cast<Cand*>(a.ws);
  count_launch();
  route_bwd_scan_kernel<T><<<dim3(kSplits, (unsigned)a.k, (unsigned)a.B), kScanThreads, 0, s>>>(a, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  count_launch();
  route_bwd_grad_kernel<T><<<dim3((unsigned)a.k, (unsigned)a.B), 32 * a.Hr, 0, s>>>(a, ws);
  return cudaGetLastError();
}

}  // namespace

size_t route_bwd_workspace_size(int64_t B, int k) {
  return ((sizeof(Cand) * (size_t)B * (size_t)k * kSplits) + 255) / 256 * 256;
}

cudaError_t launch_route_bwd(msa_dtype dt, const RouteBwdArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  return dt == MSA_F32 ? route_bwd_t<float>(a, s) : route_bwd_t<__nv_bfloat16>(a, s);
}

}  // namespace msa
