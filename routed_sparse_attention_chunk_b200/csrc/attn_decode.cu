// Step 5 of the MSA memory path for decoding: a few query tokens per batch row
// attending over [selected memory rows ++ the whole local KV]
// ("MSA x Qwen3.5" model card, "Architecture summary"; "MSA: Memory Sparse
// Attention" README, "Inference Pipeline" stage 3, sparse generation).
//
// The work is an HBM stream of K and V: with the GQA group packed as rows
// (R = G * Tq <= 16 rows per KV head) every key costs 2 R d multiply-adds, far
// below what the memory system delivers per SM, so this runs on CUDA cores and
// is shaped for bandwidth:
//   * persistent CTAs (one per SM) walk work units = (batch row, KV head,
//     key split); every split but the last holds the same number of 128-key
//     tiles;
//   * a producer thread streams K and V tiles with 2D TMA (128-byte swizzle)
//     into a ring of shared-memory stages;
//   * four compute warps: for Q K^T a lane owns one key of the tile and reads
//     its swizzled K row against the Q rows (fp32, pre-scaled, in shared
//     memory); the tile's row maxima and exp2 weights go through shared memory;
//     for P V a thread owns two output dimensions and half of the tile's keys;
//   * each unit leaves (max, sum, unnormalised O) per row in the workspace and a
//     second kernel merges the splits of every (batch row, KV head).
// Every wait is bounded; after the first expired wait the CTA stops waiting,
// finishes its loops without data, and raises MSA_FLAG_TIMEOUT.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace msa {
namespace {

using namespace sm100;

constexpr int kDH = 128;
constexpr int kKeys = 128;              // keys per tile
constexpr int kMaxRows = 16;            // R = G * Tq
constexpr int kStages = 3;
constexpr int kCompute = 128;           // compute threads (4 warps)
constexpr int kThreads = kCompute + 32; // + producer warp
constexpr uint32_t kWaitPolls = 1u << 24;

struct DecParams {
  const __nv_bfloat16* Q;
  const int32_t* mem_len;
  int32_t* err_flag;
  float* part;  // [units][R][kDH + 2]: m, l, O
  int64_t B;
  int Tq, Lloc, Hq, Hkv, Mmax, G, R;
  int NM;       // memory tiles (ceil(Mmax / kKeys)); rows past mem_len are masked
  int NL;       // local tiles (ceil(Lloc / kKeys))
  int S, tps;   // splits per (b, g) and tiles per split
  int64_t units;
  float scale_log2;
};

struct DLayout {
  static constexpr int kTile = kKeys * kDH * 2;      // one K (or V) tile
  static constexpr int kStage = 2 * kTile;
  static constexpr int kSmem = 1024 + kStages * kStage + kMaxRows * kDH * 4 + kKeys * kMaxRows * 4 +
                               4 * kMaxRows * 4 + 2 * 64 * kMaxRows * 2 * 4 + 8 * (2 * kStages) + 64;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void bar_compute() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
attn_decode_kernel(const __grid_constant__ CUtensorMap tmKm, const __grid_constant__ CUtensorMap tmVm,
                   const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmVl, DecParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* q_s = reinterpret_cast<float*>(ring + kStages * DLayout::kStage);  // [R][kDH]
  float* p_s = q_s + kMaxRows * kDH;                                        // [kKeys][R]
  float* red_s = p_s + kKeys * kMaxRows;                                    // [4 warps][R]
  float* o_s = red_s + 4 * kMaxRows;                                        // [64 pairs][R][2]
  float* l_s = o_s + 64 * kMaxRows * 2;                                     // [64][R] (sums of the upper key half)
  uint64_t* full = reinterpret_cast<uint64_t*>(l_s + 64 * kMaxRows);
  uint64_t* empty = full + kStages;
  volatile int* abort_s = reinterpret_cast<volatile int*>(empty + kStages);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = p.R;
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);  // one arrival per compute warp
    }
    *abort_s = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const int s = (int)(u % p.S);
        const int64_t bg = u / p.S;
        const int g = (int)(bg % p.Hkv);
        const int64_t b = bg / p.Hkv;
        const int t_end = min((s + 1) * p.tps, p.NM + p.NL);
        for (int t = s * p.tps; t < t_end; ++t, ++it) {
          const uint32_t st = it % kStages, round = it / kStages;
          if (!mbar_wait(&empty[st], (round & 1) ^ 1, kWaitPolls)) {
            ok = false;
            *abort_s = 1;
            break;
          }
          uint8_t* Kd = ring + st * DLayout::kStage;
          uint8_t* Vd = Kd + DLayout::kTile;
          mbar_arrive_expect_tx(&full[st], DLayout::kStage);
          const bool mem = t < p.NM;
          const CUtensorMap* mk = mem ? &tmKm : &tmKl;
          const CUtensorMap* mv = mem ? &tmVm : &tmVl;
          const int y = mem ? (int)(b * p.Mmax + t * kKeys) : (int)(b * p.Lloc + (t - p.NM) * kKeys);
          for (int dc = 0; dc < 2; ++dc) {
            tma_load_2d(Kd + dc * (kKeys * 128), mk, g * kDH + dc * 64, y, &full[st]);
            tma_load_2d(Vd + dc * (kKeys * 128), mv, g * kDH + dc * 64, y, &full[st]);
          }
        }
      }
      const uint32_t fills = it;
      for (uint32_t st = 0; st < (uint32_t)kStages && st < fills; ++st) {
        const uint32_t last = (fills - 1 - st) / kStages * kStages + st;
        if (!mbar_wait(&full[st], (last / kStages) & 1, kWaitPolls)) *abort_s = 1;
      }
    }
  } else {
    // ---------------------------------------------------------------- compute
    uint32_t it = 0;
    const int dp = tid & 63, kh = tid >> 6;  // P V: output pair dp (dims 2dp, 2dp+1), key half kh
    for (int64_t u = blockIdx.x; u < p.units; u += gridDim.x) {
      const int s = (int)(u % p.S);
      const int64_t bg = u / p.S;
      const int g = (int)(bg % p.Hkv);
      const int64_t b = bg / p.Hkv;
      int M = __ldg(p.mem_len + b);
      if (M < 0 || M > p.Mmax) {
        if (tid == 0 && s == 0 && g == 0) raise_flag(p.err_flag, MSA_FLAG_INDEX_OOB);
        M = M < 0 ? 0 : p.Mmax;
      }
      // Q rows (row r = token r / G, head g * G + r % G), fp32, scaled into the log2 domain
      bar_compute();
      for (int i = tid; i < R * kDH; i += kCompute) {
        const int r = i / kDH, col = i - r * kDH;
        const int t = r / p.G, h = g * p.G + r % p.G;
        q_s[i] = __bfloat162float(p.Q[((b * p.Tq + t) * p.Hq + h) * (int64_t)kDH + col]) * p.scale_log2;
      }
      bar_compute();
      float m_run[kMaxRows], l_run[kMaxRows], o0[kMaxRows], o1[kMaxRows];
#pragma unroll
      for (int r = 0; r < kMaxRows; ++r) {
        m_run[r] = -INFINITY;
        l_run[r] = 0.f;
        o0[r] = o1[r] = 0.f;
      }
      const int t_end = min((s + 1) * p.tps, p.NM + p.NL);
      for (int t = s * p.tps; t < t_end; ++t, ++it) {
        const uint32_t st = it % kStages, round = it / kStages;
        if (!*abort_s) {
          const bool got = __all_sync(0xffffffffu, mbar_wait(&full[st], round & 1, kWaitPolls));
          if (!got) *abort_s = 1;
        }
        const uint8_t* Kt = ring + st * DLayout::kStage;
        const uint8_t* Vt = Kt + DLayout::kTile;
        // -------- Q K^T: lane owns key kr = 32 * warp + lane
        const int kr = 32 * warp + lane;
        const bool mem = t < p.NM;
        const int key_base = mem ? t * kKeys : (t - p.NM) * kKeys;
        float sc[kMaxRows];
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) sc[r] = 0.f;
#pragma unroll 4
        for (int ch = 0; ch < kDH / 8; ++ch) {
          const int box = ch >> 3, c16 = ch & 7;
          const uint4 kv = *reinterpret_cast<const uint4*>(Kt + box * (kKeys * 128) + kr * 128 +
                                                           ((c16 ^ (kr & 7)) << 4));
          float k8[8];
          unpack(kv, k8);
#pragma unroll
          for (int r = 0; r < kMaxRows; ++r) {
            if (r < R) {
              const float4 qa = *reinterpret_cast<const float4*>(q_s + r * kDH + ch * 8);
              const float4 qb = *reinterpret_cast<const float4*>(q_s + r * kDH + ch * 8 + 4);
              sc[r] += qa.x * k8[0] + qa.y * k8[1] + qa.z * k8[2] + qa.w * k8[3] + qb.x * k8[4] + qb.y * k8[5] +
                       qb.z * k8[6] + qb.w * k8[7];
            }
          }
        }
        // mask: memory rows past mem_len, local rows past each row's causal position
        const int key = key_base + kr;
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) {
          const int pos = p.Lloc - p.Tq + r / p.G;
          const bool vis = r < R && (mem ? key < M : key <= pos);
          sc[r] = vis ? sc[r] : -INFINITY;
        }
        // tile max per row: warp reduce, then across the 4 warps through shared memory
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) {
          float v = sc[r];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0 && r < R) red_s[warp * kMaxRows + r] = v;
        }
        bar_compute();
        float corr[kMaxRows];
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) {
          if (r < R) {
            const float mt = fmaxf(fmaxf(red_s[r], red_s[kMaxRows + r]), fmaxf(red_s[2 * kMaxRows + r], red_s[3 * kMaxRows + r]));
            const float mn = fmaxf(m_run[r], mt);
            corr[r] = mn == -INFINITY ? 1.f : fast_exp2(m_run[r] - mn);
            m_run[r] = mn;
            const float pv = mn == -INFINITY ? 0.f : fast_exp2(sc[r] - mn);
            p_s[kr * kMaxRows + r] = pv;
            l_run[r] = l_run[r] * corr[r] + pv;  // this thread's keys only; summed at the end
          } else {
            corr[r] = 1.f;
          }
        }
        bar_compute();
        // -------- P V: thread owns dims (2dp, 2dp+1) over keys [64 kh, 64 kh + 64)
        const int box = dp >> 5, c16 = (dp & 31) >> 2, w2 = dp & 3;  // 16-byte chunk and 32-bit word
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) {
          o0[r] *= corr[r];
          o1[r] *= corr[r];
        }
#pragma unroll 4
        for (int j = 0; j < 64; ++j) {
          const int kk = kh * 64 + j;
          const uint32_t vw = *reinterpret_cast<const uint32_t*>(Vt + box * (kKeys * 128) + kk * 128 +
                                                                 ((c16 ^ (kk & 7)) << 4) + w2 * 4);
          const float v0 = __uint_as_float(vw << 16), v1 = __uint_as_float(vw & 0xffff0000u);
#pragma unroll
          for (int r4 = 0; r4 < kMaxRows; r4 += 4) {
            if (r4 < R) {
              const float4 pp = *reinterpret_cast<const float4*>(p_s + kk * kMaxRows + r4);
              o0[r4] += pp.x * v0;
              o1[r4] += pp.x * v1;
              o0[r4 + 1] += pp.y * v0;
              o1[r4 + 1] += pp.y * v1;
              o0[r4 + 2] += pp.z * v0;
              o1[r4 + 2] += pp.z * v1;
              o0[r4 + 3] += pp.w * v0;
              o1[r4 + 3] += pp.w * v1;
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
      // -------- unit result: l summed over all threads, O over the two key halves
#pragma unroll
      for (int r = 0; r < kMaxRows; ++r) {
        float v = l_run[r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && r < R) red_s[warp * kMaxRows + r] = v;
      }
      if (kh == 1) {
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r)
          if (r < R) {
            o_s[(dp * kMaxRows + r) * 2] = o0[r];
            o_s[(dp * kMaxRows + r) * 2 + 1] = o1[r];
          }
      }
      bar_compute();
      float* out = p.part + (size_t)u * R * (kDH + 2);
      if (kh == 0) {
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r)
          if (r < R) {
            float2 w;
            w.x = o0[r] + o_s[(dp * kMaxRows + r) * 2];
            w.y = o1[r] + o_s[(dp * kMaxRows + r) * 2 + 1];
            *reinterpret_cast<float2*>(out + r * (kDH + 2) + 2 + 2 * dp) = w;
          }
      }
      if (tid < R) {
        // every thread holds the same running max per row
        float m = -INFINITY;
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) m = r == tid ? m_run[r] : m;
        out[tid * (kDH + 2)] = m;
        out[tid * (kDH + 2) + 1] =
            red_s[tid] + red_s[kMaxRows + tid] + red_s[2 * kMaxRows + tid] + red_s[3 * kMaxRows + tid];
      }
    }
  }
  __syncthreads();
  if (tid == 0 && *abort_s) raise_flag(p.err_flag, MSA_FLAG_TIMEOUT);
}

// Merge the S splits of every (b, g) row: O = sum_s 2^(m_s - m) O_s / sum_s 2^(m_s - m) l_s.
__global__ void decode_combine_kernel(DecParams p, __nv_bfloat16* __restrict__ O, float* __restrict__ lse) {
  const int64_t bg = blockIdx.x;  // one CTA per (b, g), one warp per row
  const int g = (int)(bg % p.Hkv);
  const int64_t b = bg / p.Hkv;
  const int r = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (r >= p.R) return;
  float m = -INFINITY;
  for (int s = 0; s < p.S; ++s) m = fmaxf(m, p.part[((bg * p.S + s) * p.R + r) * (kDH + 2)]);
  float l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < p.S; ++s) {
    const float* src = p.part + ((bg * p.S + s) * p.R + r) * (kDH + 2);
    const float ms = src[0];
    const float w = ms == -INFINITY ? 0.f : fast_exp2(ms - m);
    l += w * src[1];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] += w * src[2 + lane * 4 + i];
  }
  const int t = r / p.G, h = g * p.G + r % p.G;
  const float inv = 1.f / l;
  __nv_bfloat16* dst = O + ((b * p.Tq + t) * p.Hq + h) * (int64_t)kDH + lane * 4;
  *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
  if (lse && lane == 0) lse[(b * p.Hq + h) * (int64_t)p.Tq + t] = (m + __log2f(l)) * 0.69314718055994531f;
}

struct DecodePlan {
  int R, NM, NL, S, tps;
  int64_t units;
};

DecodePlan plan(const AttnArgs& a) {
  DecodePlan d{};
  d.R = (a.Hq / a.Hkv) * a.Tq;
  d.NM = (a.Mmax + kKeys - 1) / kKeys;
  d.NL = (a.Lloc + kKeys - 1) / kKeys;
  const int T = d.NM + d.NL;
  const int64_t bg = a.B * a.Hkv;
  // enough equal units for ~8 per SM, each at least one tile; every split holds tps tiles
  int S = (int)((8LL * sm_count() + bg - 1) / bg);
  S = S < 1 ? 1 : (S > T ? T : S);
  d.tps = (T + S - 1) / S;
  d.S = (T + d.tps - 1) / d.tps;
  d.units = bg * d.S;
  return d;
}

}  // namespace

bool decode_applies(msa_dtype dt, const AttnArgs& a) {
  if (dt != MSA_BF16 || a.d != kDH || a.Hq % a.Hkv) return false;
  const int R = (a.Hq / a.Hkv) * a.Tq;
  return R <= kMaxRows && a.Tq <= 4;
}

size_t decode_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int Mmax) {
  AttnArgs a{};
  a.B = B;
  a.Tq = Tq;
  a.Lloc = Lloc;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Mmax = Mmax;
  const DecodePlan d = plan(a);
  return sizeof(float) * (size_t)d.units * d.R * (kDH + 2);
}

cudaError_t launch_attn_decode(const AttnArgs& a, cudaStream_t s) {
  const DecodePlan d = plan(a);
  const size_t need = sizeof(float) * (size_t)d.units * d.R * (kDH + 2);
  if (!a.ws || a.ws_bytes < need) return cudaErrorInvalidValue;
  CUtensorMap tkm, tvm, tkl, tvl;
  const uint64_t rowkv = (uint64_t)a.Hkv * kDH * 2;
  const int64_t mrows = a.B * (int64_t)(a.Mmax > 0 ? a.Mmax : 1);
  const void* km = a.Mmax > 0 ? a.Kmem : a.Kloc;
  const void* vm = a.Mmax > 0 ? a.Vmem : a.Vloc;
  const uint64_t mr = (uint64_t)(a.Mmax > 0 ? mrows : a.B * a.Lloc);
  if (!make_tmap_2d_bf16(&tkm, km, (uint64_t)a.Hkv * kDH, mr, rowkv, 64, kKeys) ||
      !make_tmap_2d_bf16(&tvm, vm, (uint64_t)a.Hkv * kDH, mr, rowkv, 64, kKeys) ||
      !make_tmap_2d_bf16(&tkl, a.Kloc, (uint64_t)a.Hkv * kDH, (uint64_t)(a.B * a.Lloc), rowkv, 64, kKeys) ||
      !make_tmap_2d_bf16(&tvl, a.Vloc, (uint64_t)a.Hkv * kDH, (uint64_t)(a.B * a.Lloc), rowkv, 64, kKeys))
    return cudaErrorInvalidValue;
  DecParams p;
  p.Q = reinterpret_cast<const __nv_bfloat16*>(a.Q);
  p.mem_len = a.mem_len;
  p.err_flag = a.err_flag;
  p.part = reinterpret_cast<float*>(a.ws);
  p.B = a.B;
  p.Tq = a.Tq;
  p.Lloc = a.Lloc;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.Mmax = a.Mmax;
  p.G = a.Hq / a.Hkv;
  p.R = d.R;
  p.NM = d.NM;
  p.NL = d.NL;
  p.S = d.S;
  p.tps = d.tps;
  p.units = d.units;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  cudaError_t e = cudaFuncSetAttribute(attn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DLayout::kSmem);
  if (e != cudaSuccess) return e;
  const int64_t grid = d.units < sm_count() ? d.units : sm_count();
  count_launch();
  attn_decode_kernel<<<(unsigned)grid, kThreads, DLayout::kSmem, s>>>(tkm, tvm, tkl, tvl, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  count_launch();
  decode_combine_kernel<<<(unsigned)(a.B * a.Hkv), 32 * d.R, 0, s>>>(p, reinterpret_cast<__nv_bfloat16*>(a.O), a.lse);
  return cudaGetLastError();
}

}  // namespace msa
