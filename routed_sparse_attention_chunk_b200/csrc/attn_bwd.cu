// Backward of steps 5 and 4 of the MSA memory path: the gradient of the sparse
// attention over [selected memory rows ++ causal local rows] for an upstream
// gradient dO, and the adjoint of the gather (each gathered row's gradient
// added back into its chunk).  MSA is trained end to end through this layer
// ("MSA: Memory Sparse Attention" README, "Architecture" and Figure 2 caption:
// top-k selection fused with sparse attention keeps the model differentiable);
// the pages print no gradient, so this is the exact derivative of the forward:
//     p_ij = exp(scale q_i.k_j - lse_i)        (the forward's log-sum-exp)
//     D_i  = sum_d dO_i O_i = sum_j p_ij dp_ij
//     dp_ij = dO_i . v_j      ds_ij = p_ij (dp_ij - D_i)
//     dq_i = scale sum_j ds_ij k_j
//     dk_j = scale sum_i ds_ij q_i     dv_j = sum_i p_ij dO_i
// with the sums over i running over the q-heads of a GQA group and the tokens
// that see key j.  CUDA-core kernels, fp32 arithmetic, fp32 gradients:
//   * bwd_rowdot_kernel: D_i, 16 bytes of a row per lane (and, when the
//     tensor-core dK / dV kernel splits key tiles, zeroes its outputs);
//   * dQ: on the tensor cores for the forward's tensor-core shapes
//     (attn_bwd_tc.cu), else bwd_dq_kernel: 16 rows of one KV head's group per
//     CTA, key tiles of 16 through shared memory (the forward's row layout);
//   * dK / dV: on the tensor cores for bf16, d = 128 and GQA groups of <= 8
//     heads (attn_bwd_tc.cu), else bwd_dkv_kernel: 16 keys of one KV head per
//     CTA, the rows that see them in blocks of 16 through shared memory; every
//     dK / dV row is written by exactly one CTA (rows of memory past mem_len
//     get zeros);
//   * gather_bwd_kernel: one CTA per selected document, fp32 atomic adds into
//     the chunk gradients (documents chosen by several queries accumulate).
#include <math.h>

#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace msa {

cudaError_t launch_attn_dq_tc(msa_dtype dt, const AttnBwdArgs& a, cudaStream_t s, bool* handled);

namespace {

constexpr int kRB = 16, kKT = 16, kNT = 128;  // rows, keys per tile (static smem <= 48 KB at d = 128)

// Buffers the row-dot launch zeroes (fp32, counted in float4).
struct ZeroList {
  float4* p[4];
  int64_t n[4];
};

// D_i = <dO_i, O_i> with LPR lanes per row, 16 bytes each; blocks past
// row_blocks zero the buffers of z instead.
template <typename T, int LPR>
__global__ void bwd_rowdot_kernel(const T* __restrict__ O, const T* __restrict__ dO, int64_t rows,
                                  float* __restrict__ Drow, int Tq, int Hq, int64_t row_blocks, ZeroList z) {
  if ((int64_t)blockIdx.x >= row_blocks) {
    const int64_t i0 = ((int64_t)blockIdx.x - row_blocks) * blockDim.x + threadIdx.x;
    const int64_t stride = ((int64_t)gridDim.x - row_blocks) * blockDim.x;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      for (int64_t i = i0; i < z.n[k]; i += stride) z.p[k][i] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  constexpr int VN = Vec<T>::N;
  constexpr int d = LPR * VN;
  // row w = (b, t, h) in O's layout; D is stored [B, Hq, Tq] like the lse
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / LPR;
  const int sub = threadIdx.x % LPR;
  float s = 0.f;
  if (w < rows) {
    float x[VN], y[VN];
    unpack(__ldg(reinterpret_cast<const uint4*>(O + w * d) + sub), x);
    unpack(__ldg(reinterpret_cast<const uint4*>(dO + w * d) + sub), y);
#pragma unroll
    for (int i = 0; i < VN; ++i) s = fmaf(x[i], y[i], s);
  }
#pragma unroll
  for (int o = LPR / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (sub == 0 && w < rows) {
    const int64_t h = w % Hq, t = (w / Hq) % Tq, b = w / ((int64_t)Hq * Tq);
    Drow[(b * Hq + h) * Tq + t] = s;
  }
}

// Key kk of the concatenation [memory (M rows) ++ local] for batch b, head g:
// pointer offsets of its K / V row.
template <typename T>
__device__ __forceinline__ const T* key_row(const AttnBwdArgs& a, const T* mem, const T* loc, int64_t b, int g,
                                            int kk, int M, int DH) {
  return kk < M ? mem + ((b * a.Mmax + kk) * a.Hkv + g) * (int64_t)DH
                : loc + ((b * a.Lloc + (kk - M)) * a.Hkv + g) * (int64_t)DH;
}

template <typename T, int DH>
__global__ void __launch_bounds__(kNT) bwd_dq_kernel(AttnBwdArgs a) {
  constexpr int CPT = DH / 8;
  __shared__ float Qs[kRB][DH + 4];
  __shared__ float dOs[kRB][DH + 4];
  __shared__ float Ks[kKT][DH + 1];
  __shared__ float Vs[kKT][DH + 1];
  __shared__ float dSs[kRB][kKT];
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
  const T* Q = reinterpret_cast<const T*>(a.Q);
  const T* dO = reinterpret_cast<const T*>(a.dO);
  const T* Km = reinterpret_cast<const T*>(a.Kmem);
  const T* Vm = reinterpret_cast<const T*>(a.Vmem);
  const T* Kl = reinterpret_cast<const T*>(a.Kloc);
  const T* Vl = reinterpret_cast<const T*>(a.Vloc);
  for (int i = tid; i < kRB * DH; i += kNT) {
    const int r = i / DH, col = i - r * DH, q = r0 + r;
    float qv = 0.f, dv = 0.f;
    if (q < nrows) {
      const int64_t off = ((b * a.Tq + q / group) * a.Hq + g * group + q % group) * (int64_t)DH + col;
      qv = to_f32(Q[off]);
      dv = to_f32(dO[off]);
    }
    Qs[r][col] = qv;
    dOs[r][col] = dv;
  }
  const float lse = rvalid ? a.lse[(b * a.Hq + h) * a.Tq + t] : 0.f;
  const float Dr = rvalid ? a.Drow[(b * a.Hq + h) * a.Tq + t] : 0.f;
  float dq[CPT];
#pragma unroll
  for (int c = 0; c < CPT; ++c) dq[c] = 0.f;

  for (int k0 = 0; k0 < nkeys; k0 += kKT) {
    __syncthreads();
    for (int i = tid; i < kKT * DH; i += kNT) {
      const int kr = i / DH, col = i - kr * DH, kk = k0 + kr;
      float kv = 0.f, vv = 0.f;
      if (kk < nkeys) {
        kv = to_f32(key_row(a, Km, Kl, b, g, kk, M, DH)[col]);
        vv = to_f32(key_row(a, Vm, Vl, b, g, kk, M, DH)[col]);
      }
      Ks[kr][col] = kv;
      Vs[kr][col] = vv;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kKT / 8; ++q) {
      const int kc = sub + 8 * q, kk = k0 + kc;
      float s = 0.f, dp = 0.f;
#pragma unroll 16
      for (int i = 0; i < DH; ++i) {
        s += Qs[row][i] * Ks[kc][i];
        dp += dOs[row][i] * Vs[kc][i];
      }
      const bool vis = rvalid && kk < nkeys && (kk < M || kk - M <= pos);
      const float p = vis ? expf(s * a.scale - lse) : 0.f;
      dSs[row][kc] = p * (dp - Dr);
    }
    __syncthreads();
#pragma unroll 4
    for (int kc = 0; kc < kKT; ++kc) {
      const float ds = dSs[row][kc];
#pragma unroll
      for (int c = 0; c < CPT; ++c) dq[c] += ds * Ks[kc][sub * CPT + c];
    }
  }
  if (rvalid) {
    float* out = a.dQ + ((b * a.Tq + t) * a.Hq + h) * (int64_t)DH + sub * CPT;
#pragma unroll
    for (int c = 0; c < CPT; ++c) out[c] = dq[c] * a.scale;
  }
}

template <typename T, int DH>
__global__ void __launch_bounds__(kNT) bwd_dkv_kernel(AttnBwdArgs a) {
  constexpr int CPT = DH / 8;  // dK / dV columns per thread: 8 threads per key
  __shared__ float Ks[kKT][DH + 1];
  __shared__ float Vs[kKT][DH + 1];
  __shared__ float Qs[kRB][DH + 4];
  __shared__ float dOs[kRB][DH + 4];
  __shared__ float Ps[kRB][kKT + 1];
  __shared__ float dSs[kRB][kKT + 1];
  __shared__ float lse_s[kRB], D_s[kRB];
  const int group = a.Hq / a.Hkv;
  const int g = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int tid = threadIdx.x, key = tid >> 3, sub = tid & 7;
  int M = a.mem_len[b];
  if (M < 0 || M > a.Mmax) M = M < 0 ? 0 : a.Mmax;  // flagged by bwd_dq_kernel
  // CTA x covers keys [16 x, 16 x + 16) of [memory tiles (Mmax rows) ++ local tiles]
  const int n_mem_tiles = (a.Mmax + kKT - 1) / kKT;
  const bool memt = (int)blockIdx.x < n_mem_tiles;
  const int base = memt ? blockIdx.x * kKT : ((int)blockIdx.x - n_mem_tiles) * kKT;
  const int nk = memt ? min(kKT, a.Mmax - base) : min(kKT, a.Lloc - base);  // rows of the tile
  const int nlive = memt ? max(0, min(kKT, M - base)) : nk;                 // rows that are keys
  const T* Q = reinterpret_cast<const T*>(a.Q);
  const T* dO = reinterpret_cast<const T*>(a.dO);
  const T* Kp = reinterpret_cast<const T*>(memt ? a.Kmem : a.Kloc);
  const T* Vp = reinterpret_cast<const T*>(memt ? a.Vmem : a.Vloc);
  const int64_t rows_per_b = memt ? a.Mmax : a.Lloc;
  for (int i = tid; i < kKT * DH; i += kNT) {
    const int kr = i / DH, col = i - kr * DH;
    float kv = 0.f, vv = 0.f;
    if (kr < nlive) {
      const int64_t off = ((b * rows_per_b + base + kr) * a.Hkv + g) * (int64_t)DH + col;
      kv = to_f32(Kp[off]);
      vv = to_f32(Vp[off]);
    }
    Ks[kr][col] = kv;
    Vs[kr][col] = vv;
  }
  float dk[CPT], dv[CPT];
#pragma unroll
  for (int c = 0; c < CPT; ++c) dk[c] = dv[c] = 0.f;
  // rows (t, h in group) that see this tile: every token for memory keys, tokens
  // whose position reaches the tile's first key for local ones
  const int t_first = memt ? 0 : max(0, base - (a.Lloc - a.Tq));
  const int r_begin = (nlive > 0) ? t_first * group : a.Tq * group;
  const int nrows = a.Tq * group;
  for (int r0 = r_begin; r0 < nrows; r0 += kRB) {
    __syncthreads();
    for (int i = tid; i < kRB * DH; i += kNT) {
      const int r = i / DH, col = i - r * DH, q = r0 + r;
      float qv = 0.f, dov = 0.f;
      if (q < nrows) {
        const int64_t off = ((b * a.Tq + q / group) * a.Hq + g * group + q % group) * (int64_t)DH + col;
        qv = to_f32(Q[off]);
        dov = to_f32(dO[off]);
      }
      Qs[r][col] = qv;
      dOs[r][col] = dov;
    }
    if (tid < kRB) {
      const int q = r0 + tid;
      float l = 0.f, dd = 0.f;
      if (q < nrows) {
        const int64_t li = (b * a.Hq + g * group + q % group) * a.Tq + q / group;
        l = a.lse[li];
        dd = a.Drow[li];
      }
      lse_s[tid] = l;
      D_s[tid] = dd;
    }
    __syncthreads();
    // p and ds for the 16 x 16 (row, key) pairs: 2 pairs per thread
#pragma unroll
    for (int u = 0; u < (kRB * kKT) / kNT; ++u) {
      const int pidx = tid + u * kNT, r = pidx / kKT, kc = pidx - r * kKT;
      const int q = r0 + r, tt = q / group;
      float s = 0.f, dp = 0.f;
#pragma unroll 16
      for (int i = 0; i < DH; ++i) {
        s += Qs[r][i] * Ks[kc][i];
        dp += dOs[r][i] * Vs[kc][i];
      }
      const bool vis = q < nrows && kc < nlive && (memt || base + kc <= a.Lloc - a.Tq + tt);
      const float p = vis ? expf(s * a.scale - lse_s[r]) : 0.f;
      Ps[r][kc] = p;
      dSs[r][kc] = p * (dp - D_s[r]);
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < kRB; ++r) {
      const float p = Ps[r][key], ds = dSs[r][key];
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        dv[c] += p * dOs[r][sub * CPT + c];
        dk[c] += ds * Qs[r][sub * CPT + c];
      }
    }
  }
  if (key < nk) {
    float* dKo = memt ? a.dKmem : a.dKloc;
    float* dVo = memt ? a.dVmem : a.dVloc;
    const int64_t off = ((b * rows_per_b + base + key) * a.Hkv + g) * (int64_t)DH + sub * CPT;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      dKo[off + c] = dk[c] * a.scale;
      dVo[off + c] = dv[c];
    }
  }
}

template <typename T, int DH>
cudaError_t bwd_t(const AttnBwdArgs& a, cudaStream_t s) {
  const msa_dtype dt = std::is_same<T, float>::value ? MSA_F32 : MSA_BF16;
  const DkvPlan pl = attn_dkv_tc_plan(dt, a);
  // split dK / dV tiles accumulate with atomics: zero the outputs in the row-dot launch
  ZeroList z{};
  int64_t zero_blocks = 0;
  if (pl.applies && pl.max_chunks > 1) {
    const int64_t nl = a.B * (int64_t)a.Lloc * a.Hkv * DH / 4, nm = a.B * (int64_t)a.Mmax * a.Hkv * DH / 4;
    z = ZeroList{{reinterpret_cast<float4*>(a.dKloc), reinterpret_cast<float4*>(a.dVloc),
                  reinterpret_cast<float4*>(a.dKmem), reinterpret_cast<float4*>(a.dVmem)},
                 {nl, nl, nm, nm}};
    zero_blocks = std::min<int64_t>(4 * 148, (2 * (nl + nm) + 255) / 256);
  }
  constexpr int LPR = DH / Vec<T>::N;
  const int64_t rows = a.B * a.Tq * a.Hq;
  const int64_t row_blocks = (rows * LPR + 255) / 256;
  count_launch();
  bwd_rowdot_kernel<T, LPR><<<(unsigned)(row_blocks + zero_blocks), 256, 0, s>>>(
      reinterpret_cast<const T*>(a.O), reinterpret_cast<const T*>(a.dO), rows, a.Drow, a.Tq, a.Hq, row_blocks, z);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int group = a.Hq / a.Hkv;
  bool handled = false;
  if ((e = launch_attn_dq_tc(dt, a, s, &handled)) != cudaSuccess) return e;
  if (!handled) {
    count_launch();
    bwd_dq_kernel<T, DH><<<dim3((unsigned)((a.Tq * group + kRB - 1) / kRB), (unsigned)a.Hkv, (unsigned)a.B), kNT, 0,
                           s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (pl.applies) return launch_attn_dkv_tc(dt, a, pl, s);
  const int tiles = (a.Mmax + kKT - 1) / kKT + (a.Lloc + kKT - 1) / kKT;
  count_launch();
  bwd_dkv_kernel<T, DH><<<dim3((unsigned)tiles, (unsigned)a.Hkv, (unsigned)a.B), kNT, 0, s>>>(a);
  return cudaGetLastError();
}

// grid (k, B): one CTA adds one selected document's rows back into its chunks
__global__ void gather_bwd_kernel(GatherBwdArgs a) {
  const int64_t b = blockIdx.y;
  const int r = blockIdx.x;
  int64_t start = 0;
  for (int q = 0; q < r; ++q) {
    const int32_t j = __ldg(a.topk_idx + b * a.k + q);
    if (j >= 0 && (int64_t)j < a.D) start += __ldg(a.doc_chunk_off + j + 1) - __ldg(a.doc_chunk_off + j);
  }
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
  const int ml = __ldg(a.mem_len + b);
  const int64_t n = min(ce - cs, max((int64_t)0, (int64_t)min(ml, a.Mmax) - start));
  const int64_t row = (int64_t)a.Hkv * a.d;
  for (int64_t i = threadIdx.x; i < n * row; i += blockDim.x) {
    const int64_t rr = i / row, e = i - rr * row;
    const int64_t src = (b * a.Mmax + start + rr) * row + e;
    atomicAdd(a.dKbar + (cs + rr) * row + e, __ldg(a.dKmem + src));
    atomicAdd(a.dVbar + (cs + rr) * row + e, __ldg(a.dVmem + src));
  }
}

}  // namespace

size_t attn_bwd_workspace_size(int64_t B, int Tq, int Hq) {
  return ((sizeof(float) * (size_t)B * (size_t)Hq * (size_t)Tq) + 255) / 256 * 256;
}

cudaError_t launch_attn_bwd(msa_dtype dt, const AttnBwdArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  if (dt == MSA_F32) return a.d == 64 ? bwd_t<float, 64>(a, s) : bwd_t<float, 128>(a, s);
  return a.d == 64 ? bwd_t<__nv_bfloat16, 64>(a, s) : bwd_t<__nv_bfloat16, 128>(a, s);
}

cudaError_t launch_gather_bwd(const GatherBwdArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  count_launch();
  gather_bwd_kernel<<<dim3(a.k, (unsigned)a.B), 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
