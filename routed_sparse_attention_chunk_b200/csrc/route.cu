// Step 2 of the MSA memory path: cosine routing of the query's router
// projections against the bank's pooled router keys.
//
// "MSA: Memory Sparse Attention" README, "Architecture": relevance is the
// cosine similarity between Q_r and the chunk-pooled K̄_r, mean-pooled over
// router heads, then the token-wise max; documents are then selected from the
// chunk scores (a document scores the max over its chunks).
//
//   s[b, t, c]      = (1/Hr) sum_h rq[b,t,h] rk[c,h] <Qr[b,t,h], K̄r[c,h]>
//   doc_key[b, j]   = ordered-key(max over c in j, t < Tq of s[b, t, c])
//
// with rq = 1/||Qr|| and rk = kr_rnorm (1/||K̄r|| of the stored bank).  The
// products are exact in fp32 (bf16 inputs) and every sum is fp32.
//
// This file holds the CUDA-core kernel used for fp32 banks and for shapes the
// tensor-core kernel does not take: one CTA per tile of 32 chunks, one warp per
// router head, lane = chunk, the chunk's router key held in registers.  It also
// holds the routing prelude that every scan starts from: the per-document keys
// zeroed, the chunk -> document map, and the query norms of the tensor-core scan.
#include "common.cuh"
#include "internal.h"

namespace msa {

bool route_tc_applies(const RouteArgs& a);
cudaError_t launch_route_tc(const RouteArgs& a, cudaStream_t s);

namespace {

constexpr int kRouteRows = 8;  // query rows staged per smem block

template <typename T, int DR>
__global__ void __launch_bounds__(256)
route_generic_kernel(RouteArgs a) {
  extern __shared__ float sm[];
  const int Hr = a.Hr;
  float* qs = sm;                                   // [rows][Hr][DR]
  float* rq = qs + kRouteRows * Hr * DR;            // [rows][Hr]
  float* part = rq + kRouteRows * Hr;               // [rows][Hr][32]
  float* red = part + kRouteRows * Hr * 32;         // [Hr][32]
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nthr = blockDim.x;
  const int64_t c = (int64_t)blockIdx.x * 32 + lane;
  const bool cvalid = c < a.C;

  // this lane's chunk key for head h, in registers
  float kr[DR];
  float rk = 0.f;
  {
    const T* src = reinterpret_cast<const T*>(a.Krbar) + (cvalid ? (c * Hr + h) * DR : 0);
    constexpr int VN = Vec<T>::N;
#pragma unroll
    for (int v = 0; v < DR / VN; ++v) {
      float f[VN];
      const uint4 u = cvalid ? __ldg(reinterpret_cast<const uint4*>(src) + v) : make_uint4(0, 0, 0, 0);
      unpack(u, f);
#pragma unroll
      for (int i = 0; i < VN; ++i) kr[v * VN + i] = f[i];
    }
    if (cvalid) rk = __ldg(a.kr_rnorm + c * Hr + h);
  }
  const int doc = cvalid ? __ldg(a.chunk_doc + c) : -1;
  const float invHr = 1.0f / (float)Hr;

  for (int64_t b = 0; b < a.B; ++b) {
    float mx = -INFINITY;
    for (int t0 = 0; t0 < a.Tq; t0 += kRouteRows) {
      const int nr = min(kRouteRows, a.Tq - t0);
      // stage Qr rows (fp32) and their per-head norms
      const T* q = reinterpret_cast<const T*>(a.Qr) + ((b * a.Tq + t0) * Hr) * (int64_t)DR;
      for (int i = threadIdx.x; i < kRouteRows * Hr * DR; i += nthr)
        qs[i] = i < nr * Hr * DR ? to_f32(q[i]) : 0.f;
      __syncthreads();
      for (int r = 0; r < kRouteRows; ++r) {  // warp h: norm of head h of row r
        float ss = 0.f;
        for (int i = lane; i < DR; i += 32) {
          const float v = qs[(r * Hr + h) * DR + i];
          ss += v * v;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) rq[r * Hr + h] = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
      }
      __syncthreads();
      for (int r = 0; r < nr; ++r) {
        const float4* qv = reinterpret_cast<const float4*>(qs + (r * Hr + h) * DR);
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < DR / 4; ++i) {
          const float4 w = qv[i];
          dot += w.x * kr[4 * i] + w.y * kr[4 * i + 1] + w.z * kr[4 * i + 2] + w.w * kr[4 * i + 3];
        }
        part[(r * Hr + h) * 32 + lane] = dot * rq[r * Hr + h] * rk;
      }
      __syncthreads();
      for (int r = h; r < nr; r += Hr) {
        float sum = 0.f;
        for (int g = 0; g < Hr; ++g) sum += part[(r * Hr + g) * 32 + lane];
        mx = fmaxf(mx, sum * invHr);
      }
      __syncthreads();
    }
    red[h * 32 + lane] = mx;
    __syncthreads();
    if (h == 0) {
      float v = -INFINITY;
      for (int g = 0; g < Hr; ++g) v = fmaxf(v, red[g * 32 + lane]);
      // segmented max over this warp's chunks of one document (chunks of a
      // document are contiguous), then one atomic per document segment
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float vo = __shfl_down_sync(0xffffffffu, v, o);
        const int jo = __shfl_down_sync(0xffffffffu, doc, o);
        if (lane + o < 32 && jo == doc) v = fmaxf(v, vo);
      }
      const int jprev = __shfl_up_sync(0xffffffffu, doc, 1);
      if (doc >= 0 && (lane == 0 || jprev != doc))
        atomicMax(a.doc_key + b * a.D + doc, float_to_key(v));
    }
    __syncthreads();
  }
}

template <typename T, int DR>
cudaError_t route_generic_t(const RouteArgs& a, cudaStream_t s) {
  const int threads = 32 * a.Hr;
  const size_t sm = (size_t)(kRouteRows * a.Hr * DR + kRouteRows * a.Hr + kRouteRows * a.Hr * 32 +
                             a.Hr * 32) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(route_generic_kernel<T, DR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (a.C + 31) / 32;
  if (blocks == 0) return cudaSuccess;
  count_launch();
  route_generic_kernel<T, DR><<<(unsigned)blocks, threads, sm, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

// One launch ahead of the scan: zero the document keys and the top-k counters
// that follow them, map every chunk to its owning document (one warp per 32
// chunks; offsets whose ends are not 0 and C are flagged), and for the
// tensor-core scan the inverse norms rq[r, h] = 1 / max(||Qr[r, h]||, 1e-12)
// of the bf16 query rows (one warp per row and head).  Blocks
// [0, nb_zero) zero, [nb_zero, nb_zero + nb_map) map, the rest take norms.
__global__ void __launch_bounds__(256)
route_prelude_kernel(uint32_t* __restrict__ keys, int64_t nkeys, int nb_zero, const int64_t* __restrict__ off,
                     int64_t D, int64_t C, int32_t* __restrict__ chunk_doc, int nb_map,
                     const __nv_bfloat16* __restrict__ Qr, int64_t nq, int dr, float* __restrict__ rq,
                     int32_t* err_flag) {
  // the scan may launch now: its TMA and MMA warps need nothing written here,
  // and its epilogue waits for this grid before reading any of it
  pdl_trigger();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int blk = blockIdx.x;
  if (blk < nb_zero) {
    // 16-byte stores over the aligned body of this block's range
    const int64_t per = (nkeys + nb_zero - 1) / nb_zero;
    const int64_t lo = (int64_t)blk * per, hi = min(nkeys, lo + per);
    if (lo >= hi) return;
    uint32_t* k0 = keys + lo;
    const int64_t n = hi - lo;
    const int64_t pre = min(n, (int64_t)(((16u - (reinterpret_cast<uintptr_t>(k0) & 15u)) & 15u) >> 2));
    const int64_t nv = (n - pre) >> 2;
    for (int64_t i = threadIdx.x; i < pre; i += blockDim.x) k0[i] = 0u;
    uint4* v = reinterpret_cast<uint4*>(k0 + pre);
    for (int64_t i = threadIdx.x; i < nv; i += blockDim.x) v[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t i = pre + 4 * nv + threadIdx.x; i < n; i += blockDim.x) k0[i] = 0u;
    return;
  }
  if (blk < nb_zero + nb_map) {
    const int64_t c0 = ((int64_t)(blk - nb_zero) * 8 + wib) * 32;
    if (blk == nb_zero && threadIdx.x == 0 && (__ldg(off) != 0 || __ldg(off + D) != C))
      raise_flag(err_flag, MSA_FLAG_OFFSETS);
    if (c0 >= C) return;  // whole warp
    int doc = warp_chunk_docs(off, D, C, c0, lane);
    if (doc >= D) {  // only reachable with offsets that do not end at C: never index past D
      raise_flag(err_flag, MSA_FLAG_OFFSETS);
      doc = -1;
    }
    if (c0 + lane < C) chunk_doc[c0 + lane] = doc;
    return;
  }
  const int64_t w = (int64_t)(blk - nb_zero - nb_map) * 8 + wib;
  if (w >= nq) return;
  const __nv_bfloat16* x = Qr + w * dr;
  float ss = 0.f;
  for (int i = lane; i < dr; i += 32) {
    const float v = __bfloat162float(x[i]);
    ss += v * v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) rq[w] = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
}

cudaError_t launch_route(msa_dtype dt, const RouteArgs& a, cudaStream_t s) {
  const bool tc = dt == MSA_BF16 && route_tc_applies(a);
  const int64_t nkeys = a.B * a.D + a.B;  // document keys, then the top-k counters
  const int64_t zb = (nkeys + 8191) / 8192;
  const int nb_zero = (int)(zb < 1 ? 1 : (zb > 1024 ? 1024 : zb));
  const int nb_map = (int)((a.C + 255) / 256);
  const int64_t nq = tc ? a.B * a.Tq * a.Hr : 0;
  const int64_t nb_q = (nq + 7) / 8;
  count_launch();
  route_prelude_kernel<<<(unsigned)(nb_zero + nb_map + nb_q), 256, 0, s>>>(
      a.doc_key, nkeys, nb_zero, a.doc_chunk_off, a.D, a.C, a.chunk_doc, nb_map,
      reinterpret_cast<const __nv_bfloat16*>(a.Qr), nq, a.dr, a.rq, a.err_flag);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (tc) return launch_route_tc(a, s);
  if (dt == MSA_F32)
    return a.dr == 64 ? route_generic_t<float, 64>(a, s) : route_generic_t<float, 128>(a, s);
  return a.dr == 64 ? route_generic_t<__nv_bfloat16, 64>(a, s) : route_generic_t<__nv_bfloat16, 128>(a, s);
}

}  // namespace msa
