// Step 5 of the MSA memory path: GQA softmax attention over
// [selected memory rows ++ causal local rows].
//
// "MSA x Qwen3.5" model card, "Architecture summary": full-attention MSA layers
// concatenate the top-k chunks' K/V with the local KV in sparse attention;
// "MSA: Memory Sparse Attention" README, "Architecture" (the compressed K/V are
// concatenated with the query's local K/V).  Memory rows are never masked; local
// row l is visible to query token i when l <= Lloc - Tq + i.
//
// This file holds the CUDA-core kernel (fp32 everywhere; also any bf16 shape
// the tensor-core kernels do not take) and the dispatcher.  It is a flash-style
// online softmax: a CTA owns 16 query rows of one KV head (rows are (token,
// q-head) pairs of that head's GQA group) and streams key tiles of 32 rows
// through shared memory.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace msa {

cudaError_t launch_attn_tc(msa_dtype dt, const AttnArgs& a, cudaStream_t s, bool* handled);
bool attn_tc_applies(msa_dtype dt, const AttnArgs& a);
bool decode_applies(msa_dtype dt, const AttnArgs& a);
size_t decode_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int Mmax);
size_t decode_workspace_size_smax(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int Smax);
cudaError_t launch_attn_decode(const AttnArgs& a, cudaStream_t s);

namespace {

constexpr int kRB = 16, kKT = 32, kNT = 128;

template <typename T, int DH>
__global__ void __launch_bounds__(kNT) attn_generic_kernel(AttnArgs a) {
  constexpr int CPT = DH / 8;
  __shared__ float Qs[kRB][DH + 4];
  __shared__ float Ks[kKT][DH + 1];
  __shared__ float Vs[kKT][DH];
  __shared__ float Ps[kRB][kKT];
  const int group = a.Hq / a.Hkv;
  const int g = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int r0 = blockIdx.x * kRB;
  const int nrows = a.Tq * group;
  const int tid = threadIdx.x, row = tid >> 3, sub = tid & 7;
  const int rr = r0 + row;
  const bool rvalid = rr < nrows;
  const int t = rvalid ? rr / group : 0;
  const int h = g * group + (rvalid ? rr % group : 0);
  int M = a.mem_len[b];
  if (M < 0 || M > a.Mmax) {
    if (tid == 0 && blockIdx.x == 0 && g == 0) raise_flag(a.err_flag, MSA_FLAG_INDEX_OOB);
    M = M < 0 ? 0 : a.Mmax;
  }
  const int pos = a.Lloc - a.Tq + t;
  const int tlast = (min(r0 + kRB, nrows) - 1) / group;
  const int nkeys = M + (a.Lloc - a.Tq + tlast) + 1;
  const float scale = a.scale;
  const T* Q = reinterpret_cast<const T*>(a.Q);
  const T* Km = reinterpret_cast<const T*>(a.Kmem);
  const T* Vm = reinterpret_cast<const T*>(a.Vmem);
  const T* Kl = reinterpret_cast<const T*>(a.Kloc);
  const T* Vl = reinterpret_cast<const T*>(a.Vloc);

  for (int i = tid; i < kRB * DH; i += kNT) {
    const int r = i / DH, col = i - r * DH, q = r0 + r;
    float v = 0.f;
    if (q < nrows) {
      const int tt = q / group, hh = g * group + q % group;
      v = to_f32(Q[((b * a.Tq + tt) * a.Hq + hh) * (int64_t)DH + col]);
    }
    Qs[r][col] = v * scale;
  }

  float m_run = -INFINITY, l_run = 0.f, o[CPT];
#pragma unroll
  for (int c = 0; c < CPT; ++c) o[c] = 0.f;

  for (int k0 = 0; k0 < nkeys; k0 += kKT) {
    __syncthreads();
    for (int i = tid; i < kKT * DH; i += kNT) {
      const int kr = i / DH, col = i - kr * DH, kk = k0 + kr;
      float kv = 0.f, vv = 0.f;
      if (kk < nkeys) {
        int64_t off;
        const T *kp, *vp;
        if (kk < M) {
          off = ((b * a.Mmax + kk) * a.Hkv + g) * (int64_t)DH + col;
          kp = Km; vp = Vm;
        } else {
          off = ((b * a.Lloc + (kk - M)) * a.Hkv + g) * (int64_t)DH + col;
          kp = Kl; vp = Vl;
        }
        kv = to_f32(kp[off]);
        vv = to_f32(vp[off]);
      }
      Ks[kr][col] = kv;
      Vs[kr][col] = vv;
    }
    __syncthreads();

    float sc[kKT / 8], tmax = -INFINITY;
#pragma unroll
    for (int q = 0; q < kKT / 8; ++q) {
      const int kc = sub + 8 * q, kk = k0 + kc;
      float dot = 0.f;
#pragma unroll 16
      for (int i = 0; i < DH; ++i) dot += Qs[row][i] * Ks[kc][i];
      const bool vis = rvalid && kk < nkeys && (kk < M || kk - M <= pos);
      sc[q] = vis ? dot : -INFINITY;
      tmax = fmaxf(tmax, sc[q]);
    }
#pragma unroll
    for (int o2 = 4; o2 > 0; o2 >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o2));
    const float m_new = fmaxf(m_run, tmax);
    const float corr = m_run == -INFINITY ? 0.f : expf(m_run - m_new);
    float psum = 0.f;
#pragma unroll
    for (int q = 0; q < kKT / 8; ++q) {
      const float p = sc[q] == -INFINITY ? 0.f : expf(sc[q] - m_new);
      Ps[row][sub + 8 * q] = p;
      psum += p;
    }
#pragma unroll
    for (int o2 = 4; o2 > 0; o2 >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o2);
    l_run = l_run * corr + psum;
    m_run = m_new;
#pragma unroll
    for (int c = 0; c < CPT; ++c) o[c] *= corr;
    __syncthreads();
#pragma unroll 4
    for (int kc = 0; kc < kKT; ++kc) {
      const float p = Ps[row][kc];
#pragma unroll
      for (int c = 0; c < CPT; ++c) o[c] += p * Vs[kc][sub + 8 * c];
    }
  }
  if (rvalid) {
    T* Op = reinterpret_cast<T*>(a.O) + ((b * a.Tq + t) * a.Hq + h) * (int64_t)DH;
    const float inv = 1.0f / l_run;
#pragma unroll
    for (int c = 0; c < CPT; ++c) Op[sub + 8 * c] = from_f32<T>(o[c] * inv);
    if (sub == 0 && a.lse) a.lse[(b * a.Hq + h) * (int64_t)a.Tq + t] = m_run + logf(l_run);
  }
}

template <typename T, int DH>
cudaError_t attn_generic_t(const AttnArgs& a, cudaStream_t s) {
  const int group = a.Hq / a.Hkv;
  const int64_t rows = (int64_t)a.Tq * group;
  dim3 grid((unsigned)((rows + kRB - 1) / kRB), (unsigned)a.Hkv, (unsigned)a.B);
  count_launch();
  attn_generic_kernel<T, DH><<<grid, kNT, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t attn_workspace_size(msa_dtype dt, int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, int Mmax) {
  AttnArgs a{};
  a.B = B;
  a.Tq = Tq;
  a.Lloc = Lloc;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.Mmax = Mmax;
  if (Hkv > 0 && decode_applies(dt, a)) return decode_workspace_size(B, Tq, Lloc, Hq, Hkv, Mmax);
  return 0;
}

bool attn_indexed_applies(msa_dtype dt, const AttnArgs& a) {
  return a.Hkv > 0 && a.Hq % a.Hkv == 0 && (decode_applies(dt, a) || attn_tc_applies(dt, a));
}

size_t attn_indexed_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int Smax) {
  AttnArgs a{};
  a.B = B;
  a.Tq = Tq;
  a.Lloc = Lloc;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = 128;
  if (Hkv > 0 && decode_applies(MSA_BF16, a)) return decode_workspace_size_smax(B, Tq, Lloc, Hq, Hkv, Smax);
  return 0;
}

cudaError_t launch_attn(msa_dtype dt, const AttnArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  if (a.seg_row && !attn_indexed_applies(dt, a)) return cudaErrorInvalidValue;  // only the tensor-core kernels read a plan
  if (decode_applies(dt, a)) return launch_attn_decode(a, s);
  bool handled = false;
  cudaError_t e = launch_attn_tc(dt, a, s, &handled);
  if (e != cudaSuccess || handled) return e;
  if (dt == MSA_F32) return a.d == 64 ? attn_generic_t<float, 64>(a, s) : attn_generic_t<float, 128>(a, s);
  return a.d == 64 ? attn_generic_t<__nv_bfloat16, 64>(a, s) : attn_generic_t<__nv_bfloat16, 128>(a, s);
}

}  // namespace msa
