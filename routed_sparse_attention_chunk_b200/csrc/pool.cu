// Step 1 of the MSA memory path: document-wise RoPE on K, then chunk-mean
// pooling of K, V and the router keys Kr into the memory bank.
//
// "MSA: Memory Sparse Attention" README, "Architecture" (document latent states
// K / V / K_r are chunk-mean pooled) and "Inference Pipeline" stage 1 (cache the
// chunk-pooled K̄, V̄, K̄_r); Figure 2 caption (document-wise RoPE).
//
// The work is a pure HBM stream: every raw token is read once and 1/P of that
// volume is written.  Persistent CTAs (one per SM) each own a contiguous range
// of chunks.  One producer thread follows the owning document incrementally
// and copies the token rows of K, V and Kr into a ring of shared-memory stages
// with bulk asynchronous copies (cp.async.bulk, completion counted on an
// mbarrier), running ahead across chunk boundaries; a small per-stage record
// tells the consumers which chunk the stage belongs to.  The consumer
// threads each own one column vector of the token row (8 bytes of K from the
// first half of a head together with their RoPE partners in the second half,
// or one 16-byte V / Kr vector), sum it over the chunk's tokens in fp32 from
// shared memory (the
// stage also carries the RoPE (cos, sin) rows of its token positions), and at
// the chunk's end store the mean rounded to the storage type.  The Kr threads
// also reduce the squared norm of the stored (rounded) values per head with
// warp shuffles, so kr_rnorm describes exactly the bank that routing reads.
// Every wait is bounded: on expiry the kernel raises MSA_FLAG_TIMEOUT and leaves.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace msa {
namespace {

using namespace sm100;

constexpr uint32_t kWaitPolls = 1u << 24;
constexpr int kRingBytes = 224 * 1024;  // 2 stages of 16 Qwen-shape token rows

struct PoolGeom {
  int nK, nV, nR, W;      // consumer items: Kr vectors, K pairs, V vectors
  int TOK, NS;            // tokens per stage, stages in the ring
  int rowK, rowR, rowP;   // bytes of one token's K (or V) row, Kr row, and RoPE (cos, sin) row
  int stage;              // bytes per stage
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// 8-byte vectors: the RoPE threads each own half a 16-byte vector of the low
// and of the high half of a head, so that four warps (one per SM sub-partition)
// share the rotation arithmetic, which sets the pace of a stage's consumers.
__device__ __forceinline__ void unpack8(const uint2& u, float (&f)[2]) {
  f[0] = __uint_as_float(u.x);
  f[1] = __uint_as_float(u.y);
}
__device__ __forceinline__ void unpack8(const uint2& u, float (&f)[4]) {
  f[0] = __uint_as_float(u.x << 16);  // bf16 -> fp32 is exact
  f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16);
  f[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ uint2 pack8(const float (&f)[2]) {
  return make_uint2(__float_as_uint(f[0]), __float_as_uint(f[1]));
}
__device__ __forceinline__ uint2 pack8(const float (&f)[4]) {
  return make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
}

// What the consumers need to know about one stage of the ring.
struct StageMeta {
  int64_t c;   // chunk the stage's tokens belong to
  int nt;      // tokens in this stage
  int n;       // tokens in the whole chunk
  int flags;   // kFirst: first stage of the chunk; kLast: its last stage; kEnd: no more work
};
constexpr int kFirst = 1, kLast = 2, kEnd = 4;

template <typename T>
__global__ void __launch_bounds__(512, 1) pool_kernel(PoolArgs a, PoolGeom g) {
  constexpr int VN = Vec<T>::N;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + (size_t)g.NS * g.stage);
  uint64_t* empty = full + g.NS;
  StageMeta* meta = reinterpret_cast<StageMeta*>(empty + g.NS);
  const int nconsumer_warps = (g.W + 31) / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < g.NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], nconsumer_warps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  bool timed_out = false;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // This CTA owns the contiguous chunks [c_begin, c_end); the owning document
    // is found once by a warp-wide search and then advanced incrementally.
    const int64_t per = (a.C + gridDim.x - 1) / gridDim.x;
    const int64_t c_begin = (int64_t)blockIdx.x * per, c_end = min(a.C, c_begin + per);
    const bool off_ok = __ldg(a.doc_chunk_off) == 0 && __ldg(a.doc_tok_off) == 0 &&
                        __ldg(a.doc_chunk_off + a.D) == a.C && __ldg(a.doc_tok_off + a.D) <= a.Ntok;
    int64_t j = (c_begin < c_end && off_ok) ? warp_owner_doc(a.doc_chunk_off, a.D, c_begin, lane) : 0;
    if (lane == 0) {
      if (!off_ok && blockIdx.x == 0) raise_flag(a.err_flag, MSA_FLAG_OFFSETS);
      const uint8_t* K = reinterpret_cast<const uint8_t*>(a.K);
      const uint8_t* V = reinterpret_cast<const uint8_t*>(a.V);
      const uint8_t* R = reinterpret_cast<const uint8_t*>(a.Kr);
      const uint8_t* P = reinterpret_cast<const uint8_t*>(a.rope_cs);
      uint32_t it = 0;
      for (int64_t c = off_ok ? c_begin : c_end; c < c_end && !timed_out; ++c) {
        while (j + 1 < a.D && __ldg(a.doc_chunk_off + j + 1) <= c) ++j;
        const int64_t cs = __ldg(a.doc_chunk_off + j), ce = __ldg(a.doc_chunk_off + j + 1);
        const int64_t ts = __ldg(a.doc_tok_off + j), te = __ldg(a.doc_tok_off + j + 1);
        const int64_t L = te - ts;
        if (!(c >= cs && c < ce && ts >= 0 && L >= 0 && te <= a.Ntok && (ce - cs) == (L + a.P - 1) / a.P)) {
          raise_flag(a.err_flag, MSA_FLAG_OFFSETS);
          continue;
        }
        if (L > a.max_len) {
          raise_flag(a.err_flag, MSA_FLAG_INDEX_OOB);
          continue;
        }
        const int64_t s0 = ts + (c - cs) * a.P, e0 = min(s0 + (int64_t)a.P, te);
        for (int64_t t0 = s0; t0 < e0; t0 += g.TOK, ++it) {
          const uint32_t st = it % g.NS, round = it / g.NS;
          if (!mbar_wait(&empty[st], (round & 1) ^ 1, kWaitPolls)) {
            timed_out = true;
            break;
          }
          const int nt = (int)min((int64_t)g.TOK, e0 - t0);
          meta[st] = StageMeta{c, nt, (int)(e0 - s0), (t0 == s0 ? kFirst : 0) | (t0 + nt >= e0 ? kLast : 0)};
          uint8_t* dst = ring + (size_t)st * g.stage;
          const uint32_t bK = (uint32_t)nt * g.rowK, bR = (uint32_t)nt * g.rowR, bP = (uint32_t)nt * g.rowP;
          mbar_arrive_expect_tx(&full[st], 2 * bK + bR + bP);
          bulk_load(dst, K + t0 * g.rowK, bK, &full[st]);
          bulk_load(dst + (size_t)g.TOK * g.rowK, V + t0 * g.rowK, bK, &full[st]);
          bulk_load(dst + (size_t)2 * g.TOK * g.rowK, R + t0 * g.rowR, bR, &full[st]);
          // (cos, sin) rows of the stage's positions inside the document
          bulk_load(dst + (size_t)g.TOK * (2 * g.rowK + g.rowR), P + (t0 - ts) * g.rowP, bP, &full[st]);
        }
      }
      // the end marker: a stage with no data
      if (!timed_out) {
        const uint32_t st = it % g.NS, round = it / g.NS;
        if (mbar_wait(&empty[st], (round & 1) ^ 1, kWaitPolls)) {
          meta[st] = StageMeta{-1, 0, 0, kEnd};
          mbar_arrive_expect_tx(&full[st], 0);
          ++it;
        } else {
          timed_out = true;
        }
      }
      // every copy issued must have landed before the CTA leaves
      const uint32_t fills = it;
      for (uint32_t st = 0; st < (uint32_t)g.NS && st < fills; ++st) {
        const uint32_t last = (fills - 1 - st) / g.NS * g.NS + st;
        if (!mbar_wait(&full[st], (last / g.NS) & 1, kWaitPolls)) timed_out = true;
      }
    }
  } else if (warp <= nconsumer_warps) {
    // ---------------------------------------------------------------- consumers
    constexpr int KN = VN / 2;          // elements of each half a RoPE thread owns
    const int item = threadIdx.x - 32;  // [0, nR) Kr, [nR, nR+nK) K pairs, then V; >= W idle
    const int kind = item < g.nR ? 0 : (item < g.nR + g.nK ? 1 : (item < g.W ? 2 : 3));
    const int halfv = a.d / 2 / KN;
    int off_lo = 0, off_hi = 0, region = 0, h = 0, i0 = 0;
    if (kind == 0) {
      region = 2 * g.TOK * g.rowK;
      off_lo = item * 16;
    } else if (kind == 1) {
      const int w = item - g.nR;
      h = w / halfv;
      i0 = (w - h * halfv) * KN;
      off_lo = (h * a.d + i0) * (int)sizeof(T);
      off_hi = off_lo + (a.d / 2) * (int)sizeof(T);
    } else if (kind == 2) {
      region = g.TOK * g.rowK;
      off_lo = (item - g.nR - g.nK) * 16;
    }
    const int rstride = kind == 0 ? g.rowR : g.rowK;
    const int G = a.dr / VN;  // Kr lanes per router head (a power of two <= 32)
    float acc[2 * VN];
#pragma unroll
    for (int i = 0; i < 2 * VN; ++i) acc[i] = 0.f;
    for (uint32_t it = 0;; ++it) {
      const uint32_t st = it % g.NS, round = it / g.NS;
      // the whole warp leaves together, so no warp-collective op below is split
      if (!__all_sync(0xffffffffu, mbar_wait(&full[st], round & 1, kWaitPolls))) {
        timed_out = true;
        break;
      }
      const StageMeta md = meta[st];
      if (md.flags & kEnd) break;
      if (md.flags & kFirst) {
#pragma unroll
        for (int i = 0; i < 2 * VN; ++i) acc[i] = 0.f;
      }
      const int nt = md.nt;
      const uint8_t* base = ring + (size_t)st * g.stage + region;
      if (kind == 1) {
        const uint8_t* rope = ring + (size_t)st * g.stage + (size_t)g.TOK * (2 * g.rowK + g.rowR) + i0 * 8;
#pragma unroll 4
        for (int u = 0; u < nt; ++u) {
          float xl[KN], xh[KN];
          unpack8(*reinterpret_cast<const uint2*>(base + u * rstride + off_lo), xl);
          unpack8(*reinterpret_cast<const uint2*>(base + u * rstride + off_hi), xh);
          const float4* cs4 = reinterpret_cast<const float4*>(rope + u * g.rowP);
#pragma unroll
          for (int q = 0; q < KN / 2; ++q) {
            const float4 w = cs4[q];  // (cos, sin) of pairs i0+2q and i0+2q+1
            acc[2 * q] += xl[2 * q] * w.x - xh[2 * q] * w.y;
            acc[KN + 2 * q] += xh[2 * q] * w.x + xl[2 * q] * w.y;
            acc[2 * q + 1] += xl[2 * q + 1] * w.z - xh[2 * q + 1] * w.w;
            acc[KN + 2 * q + 1] += xh[2 * q + 1] * w.z + xl[2 * q + 1] * w.w;
          }
        }
      } else if (kind != 3) {
#pragma unroll 4
        for (int u = 0; u < nt; ++u) {
          float x[VN];
          unpack(*reinterpret_cast<const uint4*>(base + u * rstride + off_lo), x);
#pragma unroll
          for (int i = 0; i < VN; ++i) acc[i] += x[i];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (!(md.flags & kLast)) continue;
      // chunk complete: mean, round to the storage type, store
      const int64_t c = md.c;
      const float fn = (float)md.n;
      float m[VN], ss = 0.f;
      if (kind == 0) {
#pragma unroll
        for (int i = 0; i < VN; ++i) m[i] = acc[i] / fn;
        const uint4 pk = pack(m);
        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(a.Krbar) + c * g.rowR + off_lo) = pk;
        unpack(pk, m);  // the stored values
#pragma unroll
        for (int i = 0; i < VN; ++i) ss += m[i] * m[i];
      } else if (kind == 1) {
        uint8_t* dst = reinterpret_cast<uint8_t*>(a.Kbar) + c * g.rowK;
        float mk[KN];
#pragma unroll
        for (int i = 0; i < KN; ++i) mk[i] = acc[i] / fn;
        *reinterpret_cast<uint2*>(dst + off_lo) = pack8(mk);
#pragma unroll
        for (int i = 0; i < KN; ++i) mk[i] = acc[KN + i] / fn;
        *reinterpret_cast<uint2*>(dst + off_hi) = pack8(mk);
      } else if (kind == 2) {
#pragma unroll
        for (int i = 0; i < VN; ++i) m[i] = acc[i] / fn;
        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(a.Vbar) + c * g.rowK + off_lo) = pack(m);
      }
      // per-head squared norm of the stored Kr: groups of G lanes (every lane
      // of the warp runs the shuffles; only Kr lanes use the result)
      for (int o = G >> 1; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (kind == 0 && a.kr_rnorm && (item % G) == 0)
        a.kr_rnorm[c * a.Hr + item / G] = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
    }
  }
  if (timed_out) raise_flag(a.err_flag, MSA_FLAG_TIMEOUT);
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
  PoolGeom g;
  g.nK = a.Hkv * (a.d / 2) / (VN / 2);
  g.nV = a.Hkv * a.d / VN;
  g.nR = a.Hr * a.dr / VN;
  g.W = g.nK + g.nV + g.nR;
  g.rowK = a.Hkv * a.d * (int)sizeof(T);
  g.rowR = a.Hr * a.dr * (int)sizeof(T);
  g.rowP = a.d * (int)sizeof(float);
  const int row = 2 * g.rowK + g.rowR + g.rowP;
  // Large stages: each bulk copy has a fixed cost in the copy engine that a
  // timeline of the ring showed dominating 8-token stages (~800 cycles per
  // stage besides the data), so two stages of 16 token rows beat four of 8.
  g.TOK = 16;
  while (g.TOK > 1 && 2 * g.TOK * row > kRingBytes) g.TOK >>= 1;
  if (g.TOK > a.P) g.TOK = a.P;
  g.stage = ((g.TOK * row + 127) / 128) * 128;
  g.NS = kRingBytes / g.stage;
  if (g.NS > 16) g.NS = 16;
  if (g.NS < 2) return cudaErrorInvalidValue;
  const int threads = 32 + ((g.W + 31) / 32) * 32;
  if (threads > 512) return cudaErrorInvalidValue;
  const size_t sm = 128 + (size_t)g.NS * g.stage + 16 * (size_t)g.NS + sizeof(StageMeta) * g.NS;
  cudaError_t e = cudaFuncSetAttribute(pool_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  if (a.C <= 0) return cudaSuccess;
  const int64_t grid = a.C < sm_count() ? a.C : sm_count();
  count_launch();
  pool_kernel<T><<<(unsigned)grid, threads, sm, s>>>(a, g);
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
