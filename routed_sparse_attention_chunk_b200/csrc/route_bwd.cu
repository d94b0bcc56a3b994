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
// Two launches: route_bwd_scan_kernel, grid (ceil(Tq / 64), k, B), recomputes
// s for the document's chunks and 64 of the query's tokens (four threads per
// token, a quarter of the router heads each, the Qr row read once per group of
// 8 chunks whose normalised K̄r rows sit in shared memory; fp32) and leaves its
// best pair in the workspace;
// route_bwd_grad_kernel, grid (k, B), one warp per router head, picks the best
// pair over the splits and adds the gradient with fp32 atomics (a token or
// chunk shared by several documents or queries accumulates).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int kTokPerBlock = 64;  // tokens per scan block (4 threads each)
constexpr int kScanThreads = 256;

struct Cand {
  float s;
  int32_t pair;  // c_rel * Tq + t; -1: none
};

__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
  return a.pair >= 0 && (b.pair < 0 || a.s > b.s || (a.s == b.s && a.pair < b.pair));
}

constexpr int kCG = 8;        // chunks per shared-memory group
constexpr int kPad = 4;       // floats after each head's row: the 4 threads of a token read
                              // 4 heads at once, and rows 528 bytes apart fall in different banks
constexpr int kMaxHD = 8 * (128 + kPad);  // Hr * (dr + kPad) at most

template <typename T>
__global__ void __launch_bounds__(kScanThreads) route_bwd_scan_kernel(RouteBwdArgs a, Cand* __restrict__ ws) {
  const int split = blockIdx.x, r = blockIdx.y;
  const int64_t b = blockIdx.z;
  __shared__ __align__(16) float khat[kCG][kMaxHD];  // K̄r[c, h, :] / |K̄r[c, h]|, head rows dr + kPad apart
  __shared__ Cand red[kScanThreads / 32];
  Cand best{-INFINITY, -1};
  const int32_t j = __ldg(a.topk_idx + b * a.k + r);
  int64_t cs = 0, n = 0;
  if (j >= 0 && (int64_t)j < a.D) {
    cs = __ldg(a.doc_chunk_off + j);
    const int64_t ce = __ldg(a.doc_chunk_off + j + 1);
    if (cs >= 0 && ce <= a.C && ce >= cs) n = ce - cs;
  }
  if (n * a.Tq > 0x7fffffffLL) {  // the pair index is int32: such a document is skipped
    if (split == 0 && threadIdx.x == 0) raise_flag(a.err_flag, MSA_FLAG_INDEX_OOB);
    n = 0;
  }
  const int HD = a.Hr * a.dr;
  const int ta = split * kTokPerBlock, tb = min(a.Tq, ta + kTokPerBlock);
  const int sub = threadIdx.x & 3, tl = threadIdx.x >> 2;
  const T* K = reinterpret_cast<const T*>(a.Krbar);
  constexpr int VN = Vec<T>::N;
  for (int64_t g0 = 0; g0 < n; g0 += kCG) {
    const int ng = (int)min((int64_t)kCG, n - g0);
    __syncthreads();  // the previous group's rows are no longer read
    // 16-byte vectors: (chunk, head) row rh, vector v of the row
    const int nv = a.dr / VN;
    for (int i = threadIdx.x; i < ng * a.Hr * nv; i += blockDim.x) {
      const int rh = i / nv, v = i - rh * nv;
      const int cc = rh / a.Hr, h = rh - cc * a.Hr;
      const int64_t c = cs + g0 + cc;
      float x[VN];
      unpack(__ldg(reinterpret_cast<const uint4*>(K + c * HD + h * a.dr) + v), x);
      const float rk = __ldg(a.kr_rnorm + c * a.Hr + h);
      float* dst = &khat[cc][h * (a.dr + kPad) + v * VN];
#pragma unroll
      for (int u = 0; u < VN; u += 4)
        *reinterpret_cast<float4*>(dst + u) = make_float4(x[u] * rk, x[u + 1] * rk, x[u + 2] * rk, x[u + 3] * rk);
    }
    __syncthreads();
    for (int t0 = ta; t0 < tb; t0 += kScanThreads / 4) {  // uniform over the block
      const int t = t0 + tl;
      const bool tv = t < tb;
      float sc[kCG];
#pragma unroll
      for (int cc = 0; cc < kCG; ++cc) sc[cc] = 0.f;
      if (tv) {
        const uint4* qv = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(a.Qr) + (b * a.Tq + t) * HD);
        for (int h = sub; h < a.Hr; h += 4) {
          float dot[kCG], nq = 0.f;
#pragma unroll
          for (int cc = 0; cc < kCG; ++cc) dot[cc] = 0.f;
          for (int v = 0; v < a.dr / VN; ++v) {
            float x[VN];
            unpack(__ldg(qv + (h * a.dr) / VN + v), x);
            const int e0 = h * (a.dr + kPad) + v * VN;
#pragma unroll
            for (int i = 0; i < VN; ++i) nq = fmaf(x[i], x[i], nq);
#pragma unroll
            for (int cc = 0; cc < kCG; ++cc) {
              if (cc < ng) {
#pragma unroll
                for (int i = 0; i < VN; i += 4) {
                  const float4 k4 = *reinterpret_cast<const float4*>(&khat[cc][e0 + i]);
                  dot[cc] = fmaf(x[i], k4.x, fmaf(x[i + 1], k4.y, fmaf(x[i + 2], k4.z, fmaf(x[i + 3], k4.w, dot[cc]))));
                }
              }
            }
          }
          const float rq = 1.f / fmaxf(sqrtf(nq), 1e-12f);
#pragma unroll
          for (int cc = 0; cc < kCG; ++cc) sc[cc] += dot[cc] * rq;
        }
      }
      // the four threads of a token hold the sums over their heads
#pragma unroll
      for (int cc = 0; cc < kCG; ++cc) {
        sc[cc] += __shfl_xor_sync(0xffffffffu, sc[cc], 1);
        sc[cc] += __shfl_xor_sync(0xffffffffu, sc[cc], 2);
      }
      if (tv && sub == 0) {
#pragma unroll
        for (int cc = 0; cc < kCG; ++cc) {
          if (cc < ng) {
            const Cand cand{sc[cc] / (float)a.Hr, (int32_t)((g0 + cc) * a.Tq + t)};
            if (better(cand, best)) best = cand;
          }
        }
      }
    }
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
    ws[(b * a.k + r) * gridDim.x + split] = best;
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
  const int nsplit = (a.Tq + kTokPerBlock - 1) / kTokPerBlock;
  for (int sp = 0; sp < nsplit; ++sp) {
    const Cand c = ws[(b * a.k + r) * nsplit + sp];
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
  const unsigned nsplit = (unsigned)((a.Tq + kTokPerBlock - 1) / kTokPerBlock);
  route_bwd_scan_kernel<T><<<dim3(nsplit, (unsigned)a.k, (unsigned)a.B), kScanThreads, 0, s>>>(a, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  count_launch();
  route_bwd_grad_kernel<T><<<dim3((unsigned)a.k, (unsigned)a.B), 32 * a.Hr, 0, s>>>(a, ws);
  return cudaGetLastError();
}

}  // namespace

size_t route_bwd_workspace_size(int64_t B, int Tq, int k) {
  const size_t nsplit = (size_t)((Tq + kTokPerBlock - 1) / kTokPerBlock);
  return ((sizeof(Cand) * (size_t)B * (size_t)k * nsplit) + 255) / 256 * 256;
}

cudaError_t launch_route_bwd(msa_dtype dt, const RouteBwdArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  return dt == MSA_F32 ? route_bwd_t<float>(a, s) : route_bwd_t<__nv_bfloat16>(a, s);
}

}  // namespace msa
