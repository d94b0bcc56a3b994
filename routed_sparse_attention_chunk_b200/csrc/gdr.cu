// The linear (DGA) layers' query path: the gated delta rule started from the
// selected documents' summed state S_ext ("MSA x Qwen3.5" model card,
// "Architecture summary": S_ext is the initial state of the query path's
// chunked gated delta rule).  The rule is that of Gated DeltaNet (Yang, Kautz
// and Hatamizadeh, "Gated Delta Networks: Improving Mamba2 with Delta Rule",
// ICLR 2025), per value head with the state h (key dim x value dim):
//     h_t = exp(g_t) (I - beta_t k_t k_t^T) h_{t-1} + beta_t k_t v_t^T,   o_t = h_t^T (scale q_t).
//
// Chunked form (C = 64 tokens; G_i the cumulative log gate inside the chunk,
// h the state at the chunk's start; with log gates <= 0 every factor kept is
// the exponential of a non-positive number, so none exceeds 1):
//   u_i + beta_i sum_{j<i} e^{G_i - G_j} (k_i . k_j) u_j = beta_i (v_i - e^{G_i} h^T k_i)
//   o_i = scale (e^{G_i} h^T q_i + sum_{j<=i} e^{G_i - G_j} (q_i . k_j) u_j)
//   h  <- e^{G_C} h + sum_j e^{G_C - G_j} k_j u_j^T
// One CTA per (32-column slice of a value head, query) walks the chunks in
// order with its fp32 slice of the state in shared memory; the chunk's products
// (K K^T, Q K^T, K h, Q h, the masked P U and K^T U) run on the CUDA cores as
// register-tiled loops over float4 rows of shared memory (row strides a
// multiple of 4 floats plus 4, so consecutive rows start on different banks),
// and the triangular system is solved by forward substitution, eight lanes per
// value column (the columns are independent).
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "msa.h"

namespace msa {
namespace {

constexpr int kC = 64;         // tokens per chunk
constexpr int kThreads = 256;

// The value columns of h evolve independently (the key-side operator
// exp(g)(I - beta k k^T) acts on every column alike), so a CTA owns a slice of
// NV value columns of one value head: four CTAs per head at d = 128, each
// repeating the chunk's K K^T and Q K^T and doing a quarter of the rest.
template <int DH, int NV>
struct GLayout {
  static constexpr int LD = DH + 4;   // row stride (floats) of the key-dim matrices
  static constexpr int LV = NV + 4;   // row stride of the value-slice matrices
  static constexpr int LC = kC + 4;   // row stride of the chunk x chunk matrices
  static constexpr int kH = DH * LV;  // state slice h [dk][NV]
  static constexpr int kK = kC * LD;  // K, Q [C][dk]
  static constexpr int kU = kC * LV;  // V / U and Q h slices [C][NV]
  static constexpr int kA = kC * LC;  // A, P [C][C]
  static constexpr int kFloats = kH + 2 * kK + 2 * kU + 2 * kA + 4 * kC;
  static constexpr int kSmem = kFloats * 4;
  static_assert(kSmem <= 232448, "shared memory of one CTA");
  static_assert(NV == 32 && kThreads == 256, "the thread tilings below");
};

struct GdrParams {
  const void *q, *k, *v;
  const float *g, *beta, *h0;
  void* o;
  float* hT;
  int64_t B;
  int T, Hk, Hv;
  float scale;
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

template <typename T, int DH, int NV>
__global__ void __launch_bounds__(kThreads, 1) gdr_chunk_kernel(GdrParams p) {
  using L = GLayout<DH, NV>;
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  float* Hs = sm;               // [DH][LV] state slice
  float* Ks = Hs + L::kH;       // [C][LD]
  float* Qs = Ks + L::kK;       // [C][LD]
  float* Us = Qs + L::kK;       // [C][LV]  (V, then beta (V - e^G K h), then U)
  float* QH = Us + L::kU;       // [C][LV]  Q h
  float* As = QH + L::kU;       // [C][LC]  beta_i e^{G_i-G_j} k_i.k_j (j < i)
  float* Ps = As + L::kA;       // [C][LC]  e^{G_i-G_j} q_i.k_j (j <= i)
  float* Gs = Ps + L::kA;       // [C] cumulative log gate
  float* Bs = Gs + kC;          // [C] beta
  float* eG = Bs + kC;          // [C] e^{G_i}
  float* dG = eG + kC;          // [C] e^{G_C - G_j}

  const int tid = threadIdx.x;
  constexpr int kSlices = DH / NV;
  const int hv = blockIdx.x / kSlices, v0 = (blockIdx.x % kSlices) * NV;  // value head, first column
  const int64_t b = blockIdx.y;
  const int hk = hv / (p.Hv / p.Hk);
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  T* o = static_cast<T*>(p.o);
  constexpr int VN = 16 / sizeof(T);  // elements per 16-byte vector
  constexpr int RK = DH / VN;          // vectors per key row
  constexpr int RVv = NV / VN;         // vectors per value-slice row
  const float* h0 = p.h0 ? p.h0 + ((int64_t)b * p.Hv + hv) * DH * DH : nullptr;

  // initial state slice (zeros when none is given)
  for (int i = tid; i < DH * NV; i += kThreads) {
    const int r = i / NV, c = i % NV;
    Hs[r * L::LV + c] = h0 ? h0[(int64_t)r * DH + v0 + c] : 0.f;
  }

  for (int t0 = 0; t0 < p.T; t0 += kC) {
    const int n = min(kC, p.T - t0);
    __syncthreads();  // the previous chunk is done with K, Q, U, Q h, A, P
    // ---- the chunk's K and Q rows (key head) and V slice (value head) in fp32; rows past n are zero
    for (int i = tid; i < kC * RK; i += kThreads) {
      const int r = i / RK, c = (i % RK) * VN;
      float fk[VN], fq[VN];
      if (r < n) {
        const int64_t tok = (int64_t)b * p.T + t0 + r;
        unpack(*reinterpret_cast<const uint4*>(k + (tok * p.Hk + hk) * DH + c), fk);
        unpack(*reinterpret_cast<const uint4*>(q + (tok * p.Hk + hk) * DH + c), fq);
      } else {
#pragma unroll
        for (int e = 0; e < VN; ++e) fk[e] = fq[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < VN; ++e) {
        Ks[r * L::LD + c + e] = fk[e];
        Qs[r * L::LD + c + e] = fq[e];
      }
    }
    for (int i = tid; i < kC * RVv; i += kThreads) {
      const int r = i / RVv, c = (i % RVv) * VN;
      float fv[VN];
      if (r < n) {
        const int64_t tok = (int64_t)b * p.T + t0 + r;
        unpack(*reinterpret_cast<const uint4*>(v + (tok * p.Hv + hv) * DH + v0 + c), fv);
      } else {
#pragma unroll
        for (int e = 0; e < VN; ++e) fv[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < VN; ++e) Us[r * L::LV + c + e] = fv[e];
    }
    // ---- cumulative log gates (one warp; two tokens per lane), write strengths
    if (tid < 32) {
      float g2[2], be[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = tid * 2 + e;
        const int64_t idx = ((int64_t)b * p.T + t0 + r) * p.Hv + hv;
        g2[e] = r < n ? p.g[idx] : 0.f;
        be[e] = r < n ? p.beta[idx] : 0.f;
      }
      float incl = g2[0] + g2[1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float x = __shfl_up_sync(0xffffffffu, incl, off);
        if (tid >= off) incl += x;
      }
      const float G1 = incl, G0 = incl - g2[1];
      const float GC = __shfl_sync(0xffffffffu, incl, 31);
      Gs[tid * 2] = G0;
      Gs[tid * 2 + 1] = G1;
      Bs[tid * 2] = be[0];
      Bs[tid * 2 + 1] = be[1];
      eG[tid * 2] = expf(G0);
      eG[tid * 2 + 1] = expf(G1);
      dG[tid * 2] = expf(GC - G0);
      dG[tid * 2 + 1] = expf(GC - G1);
    }
    __syncthreads();
    // ---- A = beta_i e^{G_i - G_j} K K^T (strictly lower), P = e^{G_i - G_j} Q K^T (lower): 4 x 4 per
    // thread; tiles wholly above the diagonal or past the chunk's last token are zero
    {
      const int i0 = (tid >> 4) * 4, j0 = (tid & 15) * 4;
      float a[4][4], pq[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) a[x][y] = pq[x][y] = 0.f;
      if (j0 <= i0 + 3 && i0 < n) {
        for (int c = 0; c < DH; c += 4) {
          float4 ki[4], qi[4], kj[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            ki[x] = ld4(Ks + (i0 + x) * L::LD + c);
            qi[x] = ld4(Qs + (i0 + x) * L::LD + c);
            kj[x] = ld4(Ks + (j0 + x) * L::LD + c);
          }
#pragma unroll
          for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              a[x][y] += ki[x].x * kj[y].x + ki[x].y * kj[y].y + ki[x].z * kj[y].z + ki[x].w * kj[y].w;
              pq[x][y] += qi[x].x * kj[y].x + qi[x].y * kj[y].y + qi[x].z * kj[y].z + qi[x].w * kj[y].w;
            }
        }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int i = i0 + x;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int j = j0 + y;
          // (above the diagonal the factor may overflow; the select drops it, no product is kept)
          const float dec = expf(Gs[i] - Gs[j]);
          As[i * L::LC + j] = j < i ? Bs[i] * dec * a[x][y] : 0.f;
          Ps[i * L::LC + j] = j <= i ? dec * pq[x][y] : 0.f;
        }
      }
    }
    // ---- K h and Q h (C x NV): 2 rows x 4 columns per thread; then the right-hand sides
    {
      const int i0 = (tid >> 3) * 2, cc = (tid & 7) * 4;
      float kh[2][4], qh[2][4];
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) kh[x][y] = qh[x][y] = 0.f;
      if (i0 < n) {
        for (int c = 0; c < DH; ++c) {
          const float4 hr = ld4(Hs + c * L::LV + cc);
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const float kv = Ks[(i0 + x) * L::LD + c], qv = Qs[(i0 + x) * L::LD + c];
            kh[x][0] = fmaf(kv, hr.x, kh[x][0]);
            kh[x][1] = fmaf(kv, hr.y, kh[x][1]);
            kh[x][2] = fmaf(kv, hr.z, kh[x][2]);
            kh[x][3] = fmaf(kv, hr.w, kh[x][3]);
            qh[x][0] = fmaf(qv, hr.x, qh[x][0]);
            qh[x][1] = fmaf(qv, hr.y, qh[x][1]);
            qh[x][2] = fmaf(qv, hr.z, qh[x][2]);
            qh[x][3] = fmaf(qv, hr.w, qh[x][3]);
          }
        }
      }
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int i = i0 + x;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          float* u = Us + i * L::LV + cc + y;
          *u = Bs[i] * (*u - eG[i] * kh[x][y]);
          QH[i * L::LV + cc + y] = qh[x][y];
        }
      }
    }
    __syncthreads();
    // ---- forward substitution u_i -= sum_{j<i} A_ij u_j: the 8 lanes of a column share the sum
    // over j (every 8th term each, then a shuffle reduction); a warp owns 4 whole columns, so the
    // rows only need the warp's own synchronisation
    {
      const int lane = tid & 31, col = (tid >> 5) * 4 + (lane >> 3), part = lane & 7;
      for (int i = 1; i < n; ++i) {
        float s0 = 0.f;
        for (int j = part; j < i; j += 8) s0 = fmaf(As[i * L::LC + j], Us[j * L::LV + col], s0);
        s0 += __shfl_xor_sync(0xffffffffu, s0, 4);
        s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
        s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
        if (part == 0) Us[i * L::LV + col] -= s0;
        __syncwarp();
      }
    }
    __syncthreads();
    // ---- o_i = scale (e^{G_i} (Q h)_i + sum_{j<=i} P_ij u_j): 2 rows x 4 columns per thread
    {
      const int i0 = (tid >> 3) * 2, cc = (tid & 7) * 4;
      if (i0 < n) {
        float acc[2][4];
#pragma unroll
        for (int x = 0; x < 2; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
        const int jmax = min(i0 + 2, n);
        for (int j = 0; j < jmax; ++j) {
          const float4 ur = ld4(Us + j * L::LV + cc);
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const float pv = Ps[(i0 + x) * L::LC + j];
            acc[x][0] = fmaf(pv, ur.x, acc[x][0]);
            acc[x][1] = fmaf(pv, ur.y, acc[x][1]);
            acc[x][2] = fmaf(pv, ur.z, acc[x][2]);
            acc[x][3] = fmaf(pv, ur.w, acc[x][3]);
          }
        }
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int i = i0 + x;
          if (i >= n) continue;
          const int64_t tok = (int64_t)b * p.T + t0 + i;
          T* orow = o + (tok * p.Hv + hv) * DH + v0 + cc;
#pragma unroll
          for (int y = 0; y < 4; ++y) orow[y] = from_f32<T>(p.scale * fmaf(eG[i], QH[i * L::LV + cc + y], acc[x][y]));
        }
      }
    }
    // ---- h <- e^{G_C} h + sum_j e^{G_C - G_j} k_j u_j^T: 4 key rows x 4 columns per thread
    {
      const int r0 = (tid >> 3) * 4, cc = (tid & 7) * 4;
      const float eC = eG[n - 1];
      float acc[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
      for (int j = 0; j < n; ++j) {
        const float dj = dG[j];
        const float4 kr = ld4(Ks + j * L::LD + r0);
        const float4 ur = ld4(Us + j * L::LV + cc);
        const float kx[4] = {dj * kr.x, dj * kr.y, dj * kr.z, dj * kr.w};
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          acc[x][0] = fmaf(kx[x], ur.x, acc[x][0]);
          acc[x][1] = fmaf(kx[x], ur.y, acc[x][1]);
          acc[x][2] = fmaf(kx[x], ur.z, acc[x][2]);
          acc[x][3] = fmaf(kx[x], ur.w, acc[x][3]);
        }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          float* h = Hs + (r0 + x) * L::LV + cc + y;
          *h = fmaf(eC, *h, acc[x][y]);
        }
    }
  }
  if (p.hT) {
    __syncthreads();
    float* hT = p.hT + ((int64_t)b * p.Hv + hv) * DH * DH;
    for (int i = tid; i < DH * NV; i += kThreads) {
      const int r = i / NV, c = i % NV;
      hT[(int64_t)r * DH + v0 + c] = Hs[r * L::LV + c];
    }
  }
}

// Few tokens (decoding): the recurrence itself, token by token.  One CTA per
// (value head, query); value column c is kept by two threads, each holding
// half of h[:, c] in registers (the columns evolve independently):
//   u = k . h[:, c];  h[:, c] = g' h[:, c] + beta k (v_c - g' u)  (g' = exp(g));  o_c = scale q . h[:, c]
// the two halves' partial dot products meet in shared memory.
constexpr int kTokenMax = 16;  // sequences up to this length take this kernel

template <typename T, int DH>
__global__ void __launch_bounds__(2 * DH) gdr_token_kernel(GdrParams p) {
  constexpr int HR = DH / 2;  // rows of h per thread
  __shared__ float ks[DH], qs[DH], part[2][DH];
  const int half = threadIdx.x / DH, c = threadIdx.x % DH, r0 = half * HR;
  const int hv = blockIdx.x;
  const int64_t b = blockIdx.y;
  const int hk = hv / (p.Hv / p.Hk);
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  T* o = static_cast<T*>(p.o);
  const float* h0 = p.h0 ? p.h0 + ((int64_t)b * p.Hv + hv) * DH * DH : nullptr;
  float h[HR];
#pragma unroll
  for (int i = 0; i < HR; ++i) h[i] = h0 ? h0[(int64_t)(r0 + i) * DH + c] : 0.f;  // a row: consecutive over c
  for (int t = 0; t < p.T; ++t) {
    const int64_t tok = (int64_t)b * p.T + t;
    const int64_t gi = tok * p.Hv + hv;
    __syncthreads();  // the previous token is done with ks, qs, part
    if (half == 0) ks[c] = to_f32(k[(tok * p.Hk + hk) * DH + c]);
    else qs[c] = to_f32(q[(tok * p.Hk + hk) * DH + c]);
    __syncthreads();
    float u = 0.f;
#pragma unroll
    for (int i = 0; i < HR; ++i) u = fmaf(ks[r0 + i], h[i], u);
    part[half][c] = u;
    __syncthreads();
    const float a = expf(p.g[gi]), be = p.beta[gi];
    const float w = be * (to_f32(v[gi * DH + c]) - a * (part[0][c] + part[1][c]));
    float oc = 0.f;
#pragma unroll
    for (int i = 0; i < HR; ++i) {
      h[i] = fmaf(a, h[i], ks[r0 + i] * w);
      oc = fmaf(qs[r0 + i], h[i], oc);
    }
    __syncthreads();  // every thread has read part[.][c] before it is rewritten
    part[half][c] = oc;
    __syncthreads();
    if (half == 0) o[gi * DH + c] = from_f32<T>(p.scale * (part[0][c] + part[1][c]));
  }
  if (p.hT) {
    float* hT = p.hT + ((int64_t)b * p.Hv + hv) * DH * DH;
#pragma unroll
    for (int i = 0; i < HR; ++i) hT[(int64_t)(r0 + i) * DH + c] = h[i];
  }
}

template <typename T, int DH>
cudaError_t launch_t(const GdrParams& p, cudaStream_t s) {
  if (p.T <= kTokenMax) {
    count_launch();
    gdr_token_kernel<T, DH><<<dim3((unsigned)p.Hv, (unsigned)p.B), 2 * DH, 0, s>>>(p);
    return cudaGetLastError();
  }
  constexpr int NV = 32;
  using L = GLayout<DH, NV>;
  cudaError_t e =
      cudaFuncSetAttribute(gdr_chunk_kernel<T, DH, NV>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  count_launch();
  gdr_chunk_kernel<T, DH, NV><<<dim3((unsigned)(p.Hv * (DH / NV)), (unsigned)p.B), kThreads, L::kSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gdr(msa_dtype dt, const void* q, const void* k, const void* v, const float* g, const float* beta,
                       int64_t B, int T, int Hk, int Hv, int d, const float* h0, float scale, void* o, float* hT,
                       cudaStream_t s) {
  if (B <= 0 || T <= 0) return cudaSuccess;
  if (d != 128) return cudaErrorInvalidValue;  // the thread tiling covers d = 128 (4-column float4 groups)
  GdrParams p{q, k, v, g, beta, h0, o, hT, B, T, Hk, Hv, scale};
  return dt == MSA_F32 ? launch_t<float, 128>(p, s) : launch_t<__nv_bfloat16, 128>(p, s);
}

}  // namespace msa
