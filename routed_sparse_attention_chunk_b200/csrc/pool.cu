// Step 1 of the MSA memory path: document-wise RoPE on K, then chunk-mean
// pooling of K, V and the router keys Kr into the memory bank.
//
// "MSA: Memory Sparse Attention" README, "Architecture" (document latent states
// K / V / K_r are chunk-mean pooled) and "Inference Pipeline" stage 1 (cache the
// chunk-pooled K̄, V̄, K̄_r); Figure 2 caption (document-wise RoPE).
//
// The work is a pure HBM stream: every raw token is read once (16-byte vector
// loads with the streaming cache hint), and 1/P of that volume is written.
// One CTA pools one chunk; thread w owns one 16-byte column vector of the
// token row (for K: one vector of the first half and its RoPE partner in the
// second half) and, when the CTA has several token groups, every TS-th token.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int kPoolMaxThreads = 512;
constexpr int kPoolUnroll = 4;

template <typename T>
__device__ __forceinline__ uint4 ld_stream(const T* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}

template <typename T>
__global__ void __launch_bounds__(kPoolMaxThreads)
pool_kernel(PoolArgs a, int nK, int nV, int nR, int TS) {
  constexpr int VN = Vec<T>::N;
  extern __shared__ float smem[];
  const int W = nK + nV + nR;
  const int tid = threadIdx.x;
  const int grp = tid / W;
  const int item = tid - grp * W;
  const bool active = grp < TS;
  const int halfv = a.d / 2 / VN;
  const int64_t rowK = (int64_t)a.Hkv * a.d, rowR = (int64_t)a.Hr * a.dr;
  float* part = smem;                                      // [TS-1][W][2*VN]
  float* npart = smem + (size_t)(TS - 1) * W * 2 * VN;     // [nR]

  if (blockIdx.x == 0 && tid == 0) {
    if (__ldg(a.doc_chunk_off) != 0 || __ldg(a.doc_tok_off) != 0 ||
        __ldg(a.doc_chunk_off + a.D) != a.C || __ldg(a.doc_tok_off + a.D) > a.Ntok)
      raise_flag(a.err_flag, MSA_FLAG_OFFSETS);
  }

  for (int64_t c = blockIdx.x; c < a.C; c += gridDim.x) {
    const int64_t j = owner_doc(a.doc_chunk_off, a.D, c);
    const int64_t cs = __ldg(a.doc_chunk_off + j), ce = __ldg(a.doc_chunk_off + j + 1);
    const int64_t ts = __ldg(a.doc_tok_off + j), te = __ldg(a.doc_tok_off + j + 1);
    const int64_t L = te - ts;
    const bool ok = c >= cs && c < ce && ts >= 0 && L >= 0 && te <= a.Ntok &&
                    (ce - cs) == (L + a.P - 1) / a.P;
    if (!ok || L > a.max_len) {  // block-uniform: depends on c only
      if (tid == 0) raise_flag(a.err_flag, ok ? MSA_FLAG_INDEX_OOB : MSA_FLAG_OFFSETS);
      continue;
    }
    const int64_t s = ts + (c - cs) * a.P;
    const int64_t e = min(s + (int64_t)a.P, te);
    const int n = (int)(e - s);

    float acc[2 * VN];
#pragma unroll
    for (int i = 0; i < 2 * VN; ++i) acc[i] = 0.f;

    if (active) {
      if (item < nK) {
        // K: vector i0.. of the first half of head h and its partner in the second half
        const int h = item / halfv, i0 = (item - h * halfv) * VN;
        const T* base = reinterpret_cast<const T*>(a.K) + h * a.d + i0;
        const int half = a.d / 2;
        for (int64_t t0 = s + grp; t0 < e; t0 += (int64_t)TS * kPoolUnroll) {
          uint4 lo[kPoolUnroll], hi[kPoolUnroll];
#pragma unroll
          for (int u = 0; u < kPoolUnroll; ++u) {
            const int64_t t = t0 + (int64_t)u * TS;
            if (t < e) {
              lo[u] = ld_stream(base + t * rowK);
              hi[u] = ld_stream(base + t * rowK + half);
            } else {
              lo[u] = hi[u] = make_uint4(0, 0, 0, 0);
            }
          }
#pragma unroll
          for (int u = 0; u < kPoolUnroll; ++u) {
            const int64_t t = t0 + (int64_t)u * TS;
            if (t < e) {
              const int p = (int)(t - ts);  // position inside the document
              const float4* cs4 =
                  reinterpret_cast<const float4*>(a.rope_cs + ((size_t)p * half + i0) * 2);
              float xl[VN], xh[VN];
              unpack(lo[u], xl);
              unpack(hi[u], xh);
#pragma unroll
              for (int q = 0; q < VN / 2; ++q) {
                const float4 w = __ldg(cs4 + q);  // (cos, sin) of pairs 2q and 2q+1
                const float c0 = w.x, s0 = w.y, c1 = w.z, s1 = w.w;
                acc[2 * q] += xl[2 * q] * c0 - xh[2 * q] * s0;
                acc[VN + 2 * q] += xh[2 * q] * c0 + xl[2 * q] * s0;
                acc[2 * q + 1] += xl[2 * q + 1] * c1 - xh[2 * q + 1] * s1;
                acc[VN + 2 * q + 1] += xh[2 * q + 1] * c1 + xl[2 * q + 1] * s1;
              }
            }
          }
        }
      } else {
        // V or Kr: plain mean of one column vector
        const bool isV = item < nK + nV;
        const int w = isV ? item - nK : item - nK - nV;
        const T* base = isV ? reinterpret_cast<const T*>(a.V) + (size_t)w * VN
                            : reinterpret_cast<const T*>(a.Kr) + (size_t)w * VN;
        const int64_t row = isV ? rowK : rowR;
        for (int64_t t0 = s + grp; t0 < e; t0 += (int64_t)TS * kPoolUnroll) {
          uint4 v[kPoolUnroll];
#pragma unroll
          for (int u = 0; u < kPoolUnroll; ++u) {
            const int64_t t = t0 + (int64_t)u * TS;
            v[u] = t < e ? ld_stream(base + t * row) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int u = 0; u < kPoolUnroll; ++u) {
            float x[VN];
            unpack(v[u], x);
#pragma unroll
            for (int i = 0; i < VN; ++i) acc[i] += x[i];
          }
        }
      }
    }

    // combine the token groups
    if (TS > 1) {
      if (active && grp > 0) {
        float* dst = part + ((size_t)(grp - 1) * W + item) * 2 * VN;
#pragma unroll
        for (int i = 0; i < 2 * VN; ++i) dst[i] = acc[i];
      }
      __syncthreads();
      if (grp == 0) {
        for (int g = 1; g < TS; ++g) {
          const float* src = part + ((size_t)(g - 1) * W + item) * 2 * VN;
#pragma unroll
          for (int i = 0; i < 2 * VN; ++i) acc[i] += src[i];
        }
      }
    }

    // mean, round to the storage type, store; Kr threads keep their squared norm part
    if (grp == 0) {
      const float fn = (float)n;
      float m[VN];
      if (item < nK) {
        const int h = item / halfv, i0 = (item - h * halfv) * VN;
        T* dst = reinterpret_cast<T*>(a.Kbar) + c * rowK + h * a.d + i0;
#pragma unroll
        for (int i = 0; i < VN; ++i) m[i] = acc[i] / fn;
        *reinterpret_cast<uint4*>(dst) = pack(m);
#pragma unroll
        for (int i = 0; i < VN; ++i) m[i] = acc[VN + i] / fn;
        *reinterpret_cast<uint4*>(dst + a.d / 2) = pack(m);
      } else if (item < nK + nV) {
        T* dst = reinterpret_cast<T*>(a.Vbar) + c * rowK + (size_t)(item - nK) * VN;
#pragma unroll
        for (int i = 0; i < VN; ++i) m[i] = acc[i] / fn;
        *reinterpret_cast<uint4*>(dst) = pack(m);
      } else {
        const int w = item - nK - nV;
        T* dst = reinterpret_cast<T*>(a.Krbar) + c * rowR + (size_t)w * VN;
#pragma unroll
        for (int i = 0; i < VN; ++i) m[i] = acc[i] / fn;
        const uint4 pk = pack(m);
        *reinterpret_cast<uint4*>(dst) = pk;
        float r[VN];
        unpack(pk, r);  // the stored (rounded) values
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < VN; ++i) ss += r[i] * r[i];
        npart[w] = ss;
      }
    }
    if (a.kr_rnorm) {
      __syncthreads();
      const int per = a.dr / VN;
      if (tid < a.Hr) {
        float ss = 0.f;
        for (int i = 0; i < per; ++i) ss += npart[tid * per + i];
        a.kr_rnorm[c * a.Hr + tid] = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
      }
    }
    __syncthreads();
  }
}

template <typename T>
__global__ void bank_rnorm_kernel(const T* __restrict__ Kb, int64_t C, int Hr, int dr,
                                  float* __restrict__ rn) {
  // one warp per (chunk, head)
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= C * Hr) return;
  const T* row = Kb + wid * dr;
  float ss = 0.f;
  for (int i = lane; i < dr; i += 32) {
    const float v = to_f32(row[i]);
    ss += v * v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) rn[wid] = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
}

template <typename T>
cudaError_t pool_t(const PoolArgs& a, cudaStream_t s) {
  constexpr int VN = Vec<T>::N;
  const int nK = a.Hkv * (a.d / 2) / VN, nV = a.Hkv * a.d / VN, nR = a.Hr * a.dr / VN;
  const int W = nK + nV + nR;
  int TS = kPoolMaxThreads / W;
  TS = TS < 1 ? 1 : (TS > 4 ? 4 : TS);
  if (TS > a.P) TS = a.P;
  const int threads = ((W * TS + 31) / 32) * 32;
  const size_t sm = ((size_t)(TS - 1) * W * 2 * VN + nR) * sizeof(float);
  if (sm > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(pool_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm);
    if (e != cudaSuccess) return e;
  }
  if (a.C <= 0) return cudaSuccess;
  const int64_t grid = a.C < 0x7fffffff ? a.C : 0x7fffffff;
  count_launch();
  pool_kernel<T><<<(unsigned)grid, threads, sm, s>>>(a, nK, nV, nR, TS);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(msa_dtype dt, const PoolArgs& a, cudaStream_t s) {
  return dt == MSA_F32 ? pool_t<float>(a, s) : pool_t<__nv_bfloat16>(a, s);
}

cudaError_t launch_bank_rnorm(msa_dtype dt, const void* Krbar, int64_t C, int Hr, int dr,
                              float* kr_rnorm, cudaStream_t s) {
  const int64_t warps = C * Hr;
  if (warps <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (warps * 32 + threads - 1) / threads;
  count_launch();
  if (dt == MSA_F32)
    bank_rnorm_kernel<float><<<(unsigned)blocks, threads, 0, s>>>(
        reinterpret_cast<const float*>(Krbar), C, Hr, dr, kr_rnorm);
  else
    bank_rnorm_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16*>(Krbar), C, Hr, dr, kr_rnorm);
  return cudaGetLastError();
}

}  // namespace msa
