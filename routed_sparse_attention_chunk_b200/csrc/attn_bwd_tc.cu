// Backward of step 5 on the 5th-generation tensor cores: dQ, dK and dV of the
// sparse attention over [selected memory rows ++ causal local rows] (the exact
// derivative of the forward; "MSA: Memory Sparse Attention" README,
// "Architecture": the layer is trained end to end through its sparse
// attention).  dQ: for a 128-row query tile (the GQA group's G q-heads x 128/G
// tokens, as in the forward) and every step j of 64 keys:
//   S = Q K_j^T and dP = dO V_j^T        (tcgen05.mma into TMEM, fp32)
//   P = exp(scale S - lse),  dS = P (dP - D)   (softmax warps, one row per
//        thread: the forward's log-sum-exp makes a row max unnecessary); dS
//        is rounded to bf16 and written back over S
//   dQ += dS K_j                          (dS as the MMA's A operand from TMEM,
//                                          K_j MN-major from its TMA tile)
// and dQ * scale is written in fp32 at the end.  S and dP have three TMEM
// buffers and two softmax warpgroups take alternate steps, so two steps are in
// the softmax while the tensor cores compute the next; the MMAs run in issue
// order, so S_{j+2} (issued after dQ_{j-1}, which reads the same buffer) never
// overwrites dS_{j-1} before it is read.  Warp roles (320 threads): warp 0 TMA
// producer, warp 1 TMEM owner + MMA issuer, warps 2..9 softmax (warpgroup 0
// even steps, 1 odd).  Every wait is bounded and ends the CTA with
// MSA_FLAG_TIMEOUT on expiry.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace msa {
namespace {

using namespace sm100;

constexpr int kRows = 128;   // MMA M: query rows per tile
constexpr int kKS = 64;      // keys per dQ step (N of S / dP, K of dQ)
constexpr int kKVStages = 4; // K / V ring of the dQ kernel
constexpr int kDqThreads = 320;
constexpr uint32_t kWaitPolls = 1u << 24;

struct DqParams {
  const int32_t* mem_len;
  int32_t* err_flag;
  const float* lse;   // [B, Hq, Tq] natural log
  const float* Drow;  // [B, Hq, Tq]
  float* dQ;          // [B, Tq, Hq, d] fp32
  int Tq, Lloc, Hq, Hkv, Mmax, G, TB, n_qblk;
  float scale, scale_log2;
};

template <int DH>
struct DqLayout {
  static constexpr int kBoxes = DH / 64;
  static constexpr int kQ = kRows * DH * 2;
  static constexpr int kK = kKS * DH * 2;   // one 64-key step of K or V
  static constexpr int kBar = 24 * 8;        // 17 barriers and the TMEM address
  static constexpr int kSmem = 1024 + 2 * kQ + 2 * kKVStages * kK + kBar;  // Q, dO, K[4], V[4]
  static constexpr uint32_t kTmemCols = 512;  // S[3], dP[3] (64 each), dQ (128)
  static_assert(kSmem <= 232448, "shared memory of one CTA");
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Barrier of the 256 softmax threads that also ANDs a predicate over them, so
// that a failed wait ends the loop for every softmax warp at once.
__device__ __forceinline__ bool bar_soft_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.b32 pi, %1, 0;\n bar.red.and.pred po, 1, 256, pi;\n"
      " selp.u32 %0, 1, 0, po;\n}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

template <int DH>
__global__ void __launch_bounds__(kDqThreads, 1)
attn_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmKm, const __grid_constant__ CUtensorMap tmVm,
                  const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmVl, DqParams p) {
  using L = DqLayout<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Qs = smem;
  uint8_t* dOs = Qs + L::kQ;
  uint8_t* Ks = dOs + L::kQ;                 // [kKVStages]
  uint8_t* Vs = Ks + kKVStages * L::kK;      // [kKVStages]
  uint64_t* bars = reinterpret_cast<uint64_t*>(Vs + kKVStages * L::kK);
  uint64_t* q_full = bars + 0;               // Q and dO landed
  uint64_t* kv_full = bars + 1;              // [kKVStages]
  uint64_t* kv_empty = bars + 1 + kKVStages; // [kKVStages] dQ MMA of the step done
  uint64_t* sp_full = bars + 1 + 2 * kKVStages;  // [3] S and dP of the buffer in TMEM
  uint64_t* ds_full = sp_full + 3;           // [3] dS written over S (128 arrivals: one warpgroup)
  uint64_t* dq_done = ds_full + 3;           // last dQ MMA done
  uint64_t* drain = dq_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = p.n_qblk - 1 - (int)blockIdx.x;  // longest blocks first
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int t0 = qb * p.TB;
  const int tlast = min(t0 + p.TB, p.Tq) - 1;
  int M = __ldg(p.mem_len + b);
  if (M < 0 || M > p.Mmax) {
    if (threadIdx.x == 0 && qb == 0 && g == 0) raise_flag(p.err_flag, MSA_FLAG_INDEX_OOB);
    M = M < 0 ? 0 : p.Mmax;
  }
  const int NM = (M + kKS - 1) / kKS;                           // memory steps
  const int T = NM + (p.Lloc - p.Tq + tlast + kKS) / kKS;       // + local steps up to the last causal key

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kKVStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&sp_full[i], 1);
      mbar_init(&ds_full[i], 128);
    }
    mbar_init(dq_done, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 3 * kKS, tQ = tmem + 6 * kKS;
  bool timed_out = false;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, 2 * L::kQ);
      for (int hh = 0; hh < p.G; ++hh)
#pragma unroll
        for (int dc = 0; dc < L::kBoxes; ++dc) {
          const int x = (g * p.G + hh) * DH + dc * 64, y = b * p.Tq + t0;
          tma_load_2d(Qs + dc * (kRows * 128) + hh * p.TB * 128, &tmQ, x, y, q_full);
          tma_load_2d(dOs + dc * (kRows * 128) + hh * p.TB * 128, &tmdO, x, y, q_full);
        }
      int j = 0;
      for (; j < T; ++j) {
        const int st = j % kKVStages;
        const bool mem = j < NM;
        const int y = mem ? b * p.Mmax + j * kKS : b * p.Lloc + (j - NM) * kKS;
        if (!mbar_wait(&kv_empty[st], ((j / kKVStages) & 1) ^ 1, kWaitPolls)) {
          timed_out = true;
          break;
        }
        mbar_arrive_expect_tx(&kv_full[st], 2 * L::kK);
#pragma unroll
        for (int dc = 0; dc < L::kBoxes; ++dc) {
          tma_load_2d(Ks + st * L::kK + dc * (kKS * 128), mem ? &tmKm : &tmKl, g * DH + dc * 64, y, &kv_full[st]);
          tma_load_2d(Vs + st * L::kK + dc * (kKS * 128), mem ? &tmVm : &tmVl, g * DH + dc * 64, y, &kv_full[st]);
        }
      }
      // drain: every copy issued must land before the CTA leaves
      if (!mbar_wait(q_full, 0, kWaitPolls)) timed_out = true;
      for (int st = 0; st < kKVStages && st < j; ++st) {
        const int last = (j - 1 - st) / kKVStages * kKVStages + st;
        if (!mbar_wait(&kv_full[st], (last / kKVStages) & 1, kWaitPolls)) timed_out = true;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kRows, kKS);
      constexpr uint32_t idQ = idesc_bf16_f32(kRows, DH, /*b_mn_major=*/true);
      const uint32_t q0 = smem_u32(Qs), o0 = smem_u32(dOs);
      // S, dP of step j into buffer j % 3
      auto issue_sp = [&](int j) -> bool {
        const int st = j % kKVStages, buf = j % 3;
        if (!mbar_wait(&kv_full[st], (j / kKVStages) & 1, kWaitPolls)) return false;
        tc_fence_after();
        const uint32_t k0 = smem_u32(Ks + st * L::kK), v0 = smem_u32(Vs + st * L::kK);
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const int box = k >> 2, kk = k & 3;
          mma_bf16_ss(tS + buf * kKS, desc_k_sw128(q0 + box * kRows * 128 + kk * 32),
                      desc_k_sw128(k0 + box * kKS * 128 + kk * 32), idS, k > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const int box = k >> 2, kk = k & 3;
          mma_bf16_ss(tP + buf * kKS, desc_k_sw128(o0 + box * kRows * 128 + kk * 32),
                      desc_k_sw128(v0 + box * kKS * 128 + kk * 32), idS, k > 0 ? 1u : 0u);
        }
        mma_commit(&sp_full[buf]);
        return true;
      };
      // dQ += dS_j K_j: A = dS_j from TMEM (16 keys of bf16 = 8 columns per MMA)
      auto issue_dq = [&](int j) {
        const int st = j % kKVStages, buf = j % 3;
        const uint32_t k0 = smem_u32(Ks + st * L::kK);
#pragma unroll
        for (int k = 0; k < kKS / 16; ++k)
          mma_bf16_ts(tQ, tS + buf * kKS + k * 8, desc_mn_sw128(k0 + k * 16 * 128, kKS * 128), idQ,
                      (j > 0 || k > 0) ? 1u : 0u);
        mma_commit(&kv_empty[st]);
      };
      bool ok = mbar_wait(q_full, 0, kWaitPolls) && issue_sp(0) && (T < 2 || issue_sp(1));
      for (int j = 0; ok && j < T; ++j) {
        if (j + 2 < T && !issue_sp(j + 2)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&ds_full[j % 3], (j / 3) & 1, kWaitPolls)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_dq(j);
      }
      if (ok) mma_commit(dq_done);
      if (!ok) timed_out = true;
      mma_commit(drain);
      if (!mbar_wait(drain, 0, kWaitPolls)) timed_out = true;
    }
  } else {
    // ---------------------------------------------------------------- softmax
    // Two warpgroups: warp w reaches TMEM lanes 32 (w % 4) ..; warpgroup `half`
    // takes steps j = half, half + 2, ... (all 64 key columns of each).
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = q * 32 + lane;
    const int hh = r / p.TB, t = t0 + r - hh * p.TB;
    const int h = g * p.G + hh;
    const bool rvalid = t < p.Tq;
    const int pos = p.Lloc - p.Tq + t;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const float nl = rvalid ? -__ldg(p.lse + ((int64_t)b * p.Hq + h) * p.Tq + t) * 1.4426950408889634f : 0.f;
    const float Dr = rvalid ? __ldg(p.Drow + ((int64_t)b * p.Hq + h) * p.Tq + t) : 0.f;
    for (int j = half; j < T; j += 2) {
      const int buf = j % 3;
      if (!__all_sync(0xffffffffu, mbar_wait(&sp_full[buf], (j / 3) & 1, kWaitPolls))) {
        timed_out = true;
        break;
      }
      tc_fence_after();
      const bool memt = j < NM;
      const int base = memt ? j * kKS : (j - NM) * kKS;
      const int lim = rvalid ? (memt ? M - base : pos - base + 1) : 0;  // columns [0, lim) are visible
      const bool whole = __all_sync(0xffffffffu, lim >= kKS);
#pragma unroll
      for (int c0 = 0; c0 < kKS; c0 += 32) {
        float s[32], dp[32];
        tmem_ld16(tS + buf * kKS + lane_off + c0, *reinterpret_cast<float(*)[16]>(&s[0]));
        tmem_ld16(tS + buf * kKS + lane_off + c0 + 16, *reinterpret_cast<float(*)[16]>(&s[16]));
        tmem_ld16(tP + buf * kKS + lane_off + c0, *reinterpret_cast<float(*)[16]>(&dp[0]));
        tmem_ld16(tP + buf * kKS + lane_off + c0 + 16, *reinterpret_cast<float(*)[16]>(&dp[16]));
        tmem_ld_wait();
        if (!whole) {  // masked columns: p = 0 and dS = 0
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c0 + c >= lim) {
              s[c] = -INFINITY;
              dp[c] = Dr;
            }
        }
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = fast_exp2(fmaf(s[2 * i], p.scale_log2, nl));
          const float p1 = fast_exp2(fmaf(s[2 * i + 1], p.scale_log2, nl));
          w[i] = pack_bf16x2(p0 * (dp[2 * i] - Dr), p1 * (dp[2 * i + 1] - Dr));
        }
        tmem_st16(tS + buf * kKS + lane_off + c0 / 2, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ds_full[buf]);
    }
    // dQ * scale: warpgroup `half` writes columns [64 half, 64 half + 64) of its rows
    if (!timed_out && __all_sync(0xffffffffu, mbar_wait(dq_done, 0, kWaitPolls))) {
      tc_fence_after();
      float* out = p.dQ + (((int64_t)b * p.Tq + t) * p.Hq + h) * DH + half * (DH / 2);
#pragma unroll
      for (int c = 0; c < DH / 2; c += 32) {
        float o[32];
        tmem_ld16(tQ + lane_off + half * (DH / 2) + c, *reinterpret_cast<float(*)[16]>(&o[0]));
        tmem_ld16(tQ + lane_off + half * (DH / 2) + c + 16, *reinterpret_cast<float(*)[16]>(&o[16]));
        tmem_ld_wait();
        if (rvalid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(out + c + i) =
                make_float4(o[i] * p.scale, o[i + 1] * p.scale, o[i + 2] * p.scale, o[i + 3] * p.scale);
        }
      }
    } else {
      timed_out = true;
    }
  }

  if (timed_out) raise_flag(p.err_flag, MSA_FLAG_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// dK and dV.  One CTA per 128-key tile of one (KV head, batch row) and one
// chunk of the query steps that see the keys (a long range is split so that
// every SM gets a similar share); per step of 64 query rows (the GQA group's G
// heads x 64/G tokens):
//   S^T = K Q^T, dP^T = V dO^T          (keys are the MMA's M, one TMEM lane each)
//   P^T = exp(scale S^T - lse), dS^T = P^T (dP^T - D)   (softmax warps, one key per
//        thread, the rows' lse and D staged in shared memory); both rounded to
//        bf16 and written back over S^T and dP^T
//   dV += P^T dO,  dK += dS^T Q          (A from TMEM, dO / Q MN-major from TMA)
// S^T and dP^T have two TMEM buffers each, so the tensor cores compute step
// n+1 while the softmax warps work on step n; the MMAs of step n+1 are issued
// after step n-1's dV / dK, which read the same buffer, and the MMAs run in
// issue order.  Q / dO come through a 4-deep TMA ring.  dK * scale and dV are
// written in fp32 at the end: stored when the tile's query range is one chunk
// (rows that are not keys, memory rows past mem_len, get zeros), else added
// with fp32 atomics onto outputs the row-dot kernel zeroed first.
constexpr int kQS = 64;       // query rows per step (N of S^T / dP^T, K of dV / dK)
constexpr int kQStages = 4;   // Q / dO ring
constexpr int kDkvThreads = 320;  // producer, MMA issuer, two softmax warpgroups

struct DkvParams {
  const int32_t* mem_len;
  int32_t* err_flag;
  const float* lse;
  const float* Drow;
  float *dKm, *dVm, *dKl, *dVl;  // fp32 outputs
  int Tq, Lloc, Hq, Hkv, Mmax, G, TB2, n_qstep, n_mem_tiles, chunk, max_chunks;
  float scale, scale_log2;
};

template <int DH>
struct DkvLayout {
  static constexpr int kBoxes = DH / 64;
  static constexpr int kT = 128 * DH * 2;   // one 128-row bf16 tile (K or V)
  static constexpr int kQ = kQS * DH * 2;   // one 64-row step of Q or dO
  static constexpr int kRed = 2 * 2 * kQS * 4;  // [2 buffers][lse, D][64 rows]
  static constexpr int kBar = 16 * 8;
  static constexpr int kSmem = 1024 + 2 * kT + 2 * kQStages * kQ + kRed + kBar;  // K, V, Q[4], dO[4]
  static constexpr uint32_t kTmemCols = 512;  // S^T[2], dP^T[2] (64 each), dK, dV (128 each)
  static_assert(kSmem <= 232448, "shared memory of one CTA");
};

template <int DH>
__global__ void __launch_bounds__(kDkvThreads, 1)
attn_dkv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                   const __grid_constant__ CUtensorMap tmKm, const __grid_constant__ CUtensorMap tmVm,
                   const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmVl, DkvParams p) {
  using L = DkvLayout<DH>;
  const int tile = (int)blockIdx.x / p.max_chunks, ck = (int)blockIdx.x % p.max_chunks;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  int M = __ldg(p.mem_len + b);
  if (M < 0 || M > p.Mmax) M = M < 0 ? 0 : p.Mmax;  // flagged by the dQ kernel
  const bool memt = tile < p.n_mem_tiles;
  const int base = memt ? tile * 128 : (tile - p.n_mem_tiles) * 128;
  const int nk = memt ? min(128, p.Mmax - base) : min(128, p.Lloc - base);   // rows of the tile
  const int nlive = memt ? max(0, min(128, M - base)) : nk;                  // rows that are keys
  // query steps that see the keys: all for memory keys; local key l is seen from
  // token l - (Lloc - Tq) on
  const int tfirst = memt ? 0 : max(0, base - (p.Lloc - p.Tq));
  const int s0 = tfirst / p.TB2;
  const int ns_all = nlive > 0 ? p.n_qstep - s0 : 0;
  const int nchunks = (ns_all + p.chunk - 1) / p.chunk;
  if (ck >= max(nchunks, 1)) return;  // uniform over the CTA, before any barrier or TMEM
  const bool split = nchunks > 1;
  const int sA = s0 + ck * p.chunk;
  const int NS = ns_all > 0 ? min(p.chunk, ns_all - ck * p.chunk) : 0;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Ks = smem;
  uint8_t* Vs = Ks + L::kT;
  uint8_t* Qs = Vs + L::kT;                 // [kQStages]
  uint8_t* dOs = Qs + kQStages * L::kQ;     // [kQStages]
  float* red = reinterpret_cast<float*>(dOs + kQStages * L::kQ);  // [2][lse, D][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red) + L::kRed);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;               // [kQStages]
  uint64_t* q_empty = bars + 1 + kQStages;   // [kQStages] dV / dK MMAs of the step done
  uint64_t* sp_full = bars + 1 + 2 * kQStages;  // [2] S^T, dP^T of the buffer in TMEM
  uint64_t* pd_full = sp_full + 2;           // [2] P^T, dS^T written (256 arrivals)
  uint64_t* acc_done = pd_full + 2;
  uint64_t* drain = acc_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sp_full[i], 1);
      mbar_init(&pd_full[i], 256);
    }
    mbar_init(acc_done, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 2 * kQS, tK = tmem + 4 * kQS, tV = tmem + 4 * kQS + 128;
  bool timed_out = false;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && NS > 0) {
      const int y = memt ? b * p.Mmax + base : b * p.Lloc + base;
      mbar_arrive_expect_tx(kv_full, 2 * L::kT);
#pragma unroll
      for (int dc = 0; dc < L::kBoxes; ++dc) {
        tma_load_2d(Ks + dc * (128 * 128), memt ? &tmKm : &tmKl, g * DH + dc * 64, y, kv_full);
        tma_load_2d(Vs + dc * (128 * 128), memt ? &tmVm : &tmVl, g * DH + dc * 64, y, kv_full);
      }
      int n = 0;
      for (; n < NS; ++n) {
        const int st = n % kQStages;
        if (!mbar_wait(&q_empty[st], ((n / kQStages) & 1) ^ 1, kWaitPolls)) {
          timed_out = true;
          break;
        }
        const int t0 = (sA + n) * p.TB2;
        mbar_arrive_expect_tx(&q_full[st], 2 * L::kQ);
        for (int hh = 0; hh < p.G; ++hh)
#pragma unroll
          for (int dc = 0; dc < L::kBoxes; ++dc) {
            const int x = (g * p.G + hh) * DH + dc * 64, yq = b * p.Tq + t0;
            tma_load_2d(Qs + st * L::kQ + dc * (kQS * 128) + hh * p.TB2 * 128, &tmQ, x, yq, &q_full[st]);
            tma_load_2d(dOs + st * L::kQ + dc * (kQS * 128) + hh * p.TB2 * 128, &tmdO, x, yq, &q_full[st]);
          }
      }
      // drain: every copy issued must land before the CTA leaves
      if (!mbar_wait(kv_full, 0, kWaitPolls)) timed_out = true;
      for (int st = 0; st < kQStages && st < n; ++st) {
        const int last = (n - 1 - st) / kQStages * kQStages + st;
        if (!mbar_wait(&q_full[st], (last / kQStages) & 1, kWaitPolls)) timed_out = true;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && NS > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, kQS);
      constexpr uint32_t idA = idesc_bf16_f32(128, DH, /*b_mn_major=*/true);
      const uint32_t k0 = smem_u32(Ks), v0 = smem_u32(Vs);
      // S^T, dP^T of step n into buffer n & 1
      auto issue_sp = [&](int n) -> bool {
        const int st = n % kQStages, buf = n & 1;
        if (!mbar_wait(&q_full[st], (n / kQStages) & 1, kWaitPolls)) return false;
        tc_fence_after();
        const uint32_t q0 = smem_u32(Qs + st * L::kQ), o0 = smem_u32(dOs + st * L::kQ);
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const int box = k >> 2, kk = k & 3;
          mma_bf16_ss(tS + buf * kQS, desc_k_sw128(k0 + box * 128 * 128 + kk * 32),
                      desc_k_sw128(q0 + box * kQS * 128 + kk * 32), idS, k > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const int box = k >> 2, kk = k & 3;
          mma_bf16_ss(tP + buf * kQS, desc_k_sw128(v0 + box * 128 * 128 + kk * 32),
                      desc_k_sw128(o0 + box * kQS * 128 + kk * 32), idS, k > 0 ? 1u : 0u);
        }
        mma_commit(&sp_full[buf]);
        return true;
      };
      // dV += P^T dO, dK += dS^T Q for step n (A from TMEM: 16 query rows of bf16 = 8 columns)
      auto issue_acc = [&](int n) {
        const int st = n % kQStages, buf = n & 1;
        const uint32_t q0 = smem_u32(Qs + st * L::kQ), o0 = smem_u32(dOs + st * L::kQ);
#pragma unroll
        for (int k = 0; k < kQS / 16; ++k) {
          mma_bf16_ts(tV, tS + buf * kQS + k * 8, desc_mn_sw128(o0 + k * 16 * 128, kQS * 128), idA,
                      (n > 0 || k > 0) ? 1u : 0u);
          mma_bf16_ts(tK, tP + buf * kQS + k * 8, desc_mn_sw128(q0 + k * 16 * 128, kQS * 128), idA,
                      (n > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&q_empty[st]);
      };
      bool ok = mbar_wait(kv_full, 0, kWaitPolls) && issue_sp(0);
      for (int n = 0; ok && n < NS; ++n) {
        if (n + 1 < NS && !issue_sp(n + 1)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&pd_full[n & 1], (n >> 1) & 1, kWaitPolls)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_acc(n);
      }
      if (ok) mma_commit(acc_done);
      if (!ok) timed_out = true;
      mma_commit(drain);
      if (!mbar_wait(drain, 0, kWaitPolls)) timed_out = true;
    }
  } else {
    // ---------------------------------------------------------------- softmax (one key per thread)
    // Two warpgroups: warp w reaches TMEM lanes 32 (w % 4) ..; warpgroup `half`
    // takes query columns [32 half, 32 half + 32) of every step.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int kr = q * 32 + lane;  // this thread's key row of the tile (TMEM lane)
    const int tid = threadIdx.x - 64;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const bool key_live = kr < nlive;
    const int key = base + kr;
    const int tmin = memt ? INT_MIN : key - (p.Lloc - p.Tq);  // first token that sees the key
    // the tile's last key is seen from this token on (every key of the tile visible)
    const int tall = memt ? 0 : base + 127 - (p.Lloc - p.Tq);
    // threads 0..63 stage -lse * log2(e) of the step's rows, 64..127 their D; the
    // value of step n+1 is loaded while step n is processed
    const int sr = tid & (kQS - 1);
    const int shh = sr / p.TB2;
    const int64_t srow = ((int64_t)b * p.Hq + g * p.G + shh) * p.Tq;
    auto stage_load = [&](int n) -> float {
      const int t = (sA + n) * p.TB2 + sr - shh * p.TB2;
      if (tid >= 2 * kQS || t >= p.Tq) return 0.f;
      return tid < kQS ? -__ldg(p.lse + srow + t) * 1.4426950408889634f : __ldg(p.Drow + srow + t);
    };
    float staged = NS > 0 ? stage_load(0) : 0.f;
    const int c0 = half * 32;
    for (int n = 0; n < NS; ++n) {
      const int buf = n & 1;
      const int t0 = (sA + n) * p.TB2;
      float* rl = red + buf * (2 * kQS);
      if (tid < 2 * kQS) rl[tid] = staged;  // [lse(64), D(64)]
      if (n + 1 < NS) staged = stage_load(n + 1);
      // the staging barrier doubles as a vote on the wait, so the warps leave together
      const bool okw = __all_sync(0xffffffffu, mbar_wait(&sp_full[buf], (n >> 1) & 1, kWaitPolls));
      if (!bar_soft_and(okw)) {
        timed_out = true;
        break;
      }
      tc_fence_after();
      const bool full = nlive == 128 && t0 + p.TB2 <= p.Tq && tall <= t0;
      const float4* rl4 = reinterpret_cast<const float4*>(rl);
      float s[32], dp[32];
      tmem_ld16(tS + buf * kQS + lane_off + c0, *reinterpret_cast<float(*)[16]>(&s[0]));
      tmem_ld16(tS + buf * kQS + lane_off + c0 + 16, *reinterpret_cast<float(*)[16]>(&s[16]));
      tmem_ld16(tP + buf * kQS + lane_off + c0, *reinterpret_cast<float(*)[16]>(&dp[0]));
      tmem_ld16(tP + buf * kQS + lane_off + c0 + 16, *reinterpret_cast<float(*)[16]>(&dp[16]));
      tmem_ld_wait();
      if (!full) {  // masked step: the diagonal, a ragged end, memory rows past mem_len
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int t = t0 + ((c0 + c) & (p.TB2 - 1));
          if (!(key_live && t < p.Tq && t >= tmin)) {
            s[c] = -INFINITY;  // p = 0
            dp[c] = 0.f;       // and dS = 0 even where the masked row's dP is not finite
          }
        }
      }
      uint32_t wp[16], wd[16];
#pragma unroll
      for (int i4 = 0; i4 < 8; ++i4) {
        const float4 l4 = rl4[(c0 >> 2) + i4], d4 = rl4[(kQS >> 2) + (c0 >> 2) + i4];
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
        float pr[4], ds[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = 4 * i4 + u;
          pr[u] = fast_exp2(fmaf(s[c], p.scale_log2, lv[u]));
          ds[u] = pr[u] * (dp[c] - dv[u]);
        }
        wp[2 * i4] = pack_bf16x2(pr[0], pr[1]);
        wp[2 * i4 + 1] = pack_bf16x2(pr[2], pr[3]);
        wd[2 * i4] = pack_bf16x2(ds[0], ds[1]);
        wd[2 * i4 + 1] = pack_bf16x2(ds[2], ds[3]);
      }
      tmem_st16(tS + buf * kQS + lane_off + c0 / 2, wp);
      tmem_st16(tP + buf * kQS + lane_off + c0 / 2, wd);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&pd_full[buf]);
    }
    // outputs: dK * scale (warpgroup 0), dV (warpgroup 1), fp32
    const bool got = NS > 0 && !timed_out && __all_sync(0xffffffffu, mbar_wait(acc_done, 0, kWaitPolls));
    if (NS > 0 && !got) timed_out = true;
    // the TMEM loads are warp-collective (got is uniform); only the stores depend on the lane.
    // A split tile adds onto zeroed outputs, so its non-key rows and a timed-out CTA add nothing.
    const bool write = kr < nk && (!split || (got && key_live));
    float* out = (half == 0 ? (memt ? p.dKm : p.dKl) : (memt ? p.dVm : p.dVl)) +
                 (((int64_t)b * (memt ? p.Mmax : p.Lloc) + key) * p.Hkv + g) * DH;
    const uint32_t tacc = half == 0 ? tK : tV;
    if (got) tc_fence_after();
    const float m = half == 0 ? p.scale : 1.f;
#pragma unroll
    for (int c = 0; c < DH; c += 32) {
      float o[32];
      if (got) {
        tmem_ld16(tacc + lane_off + c, *reinterpret_cast<float(*)[16]>(&o[0]));
        tmem_ld16(tacc + lane_off + c + 16, *reinterpret_cast<float(*)[16]>(&o[16]));
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
      }
      if (write) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 v = key_live ? make_float4(o[i] * m, o[i + 1] * m, o[i + 2] * m, o[i + 3] * m)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
          if (split)
            atomicAdd(reinterpret_cast<float4*>(out + c + i), v);
          else
            *reinterpret_cast<float4*>(out + c + i) = v;
        }
      }
    }
  }

  if (timed_out) raise_flag(p.err_flag, MSA_FLAG_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace

// Work split of the tensor-core dK / dV kernel: 64-row query steps per CTA
// ("chunk") and the most chunks any key tile has.  Shapes: bf16, d = 128, a
// GQA group of G <= 8 heads dividing 64 rows into blocks of >= 8 tokens.
DkvPlan attn_dkv_tc_plan(msa_dtype dt, const AttnBwdArgs& a) {
  DkvPlan pl{false, 0, 0};
  if (dt != MSA_BF16 || a.d != 128 || a.Hkv < 1) return pl;
  const int G = a.Hq / a.Hkv;
  if (G < 1 || kQS % G != 0 || kQS / G < 8 || a.B > 65535 || a.Hkv > 65535) return pl;
  const int TB2 = kQS / G;
  const int n_qstep = (a.Tq + TB2 - 1) / TB2;
  // 64-row steps of all key tiles of one (head, batch row): memory tiles see every
  // step; local tile i from the token that sees its first key on
  int64_t steps = (int64_t)((a.Mmax + 127) / 128) * n_qstep;
  for (int base = 0; base < a.Lloc; base += 128) steps += n_qstep - std::max(0, base - (a.Lloc - a.Tq)) / TB2;
  steps *= (int64_t)a.Hkv * a.B;
  // about six CTAs' worth per SM, no chunk under 8 steps
  const int64_t target = (steps + 6 * 148 - 1) / (6 * 148);
  pl.chunk = (int)std::min<int64_t>(n_qstep, std::max<int64_t>(8, target));
  pl.max_chunks = (n_qstep + pl.chunk - 1) / pl.chunk;
  const int tiles = (a.Mmax + 127) / 128 + (a.Lloc + 127) / 128;
  if ((int64_t)tiles * pl.max_chunks > 0x7fffffff) return pl;
  pl.applies = true;
  return pl;
}

cudaError_t launch_attn_dkv_tc(msa_dtype dt, const AttnBwdArgs& a, const DkvPlan& pl, cudaStream_t s) {
  if (!pl.applies) return cudaErrorInvalidValue;
  constexpr int DH = 128;
  using L = DkvLayout<DH>;
  const int G = a.Hq / a.Hkv;
  const int TB2 = kQS / G;
  CUtensorMap tq, tdo, tkm, tvm, tkl, tvl;
  const uint64_t rowkv = (uint64_t)a.Hkv * DH * 2;
  const int64_t mrows = a.B * (int64_t)(a.Mmax > 0 ? a.Mmax : 1);
  if (!make_tmap_2d_bf16(&tq, a.Q, (uint64_t)a.Hq * DH, (uint64_t)(a.B * a.Tq), (uint64_t)a.Hq * DH * 2, 64, TB2) ||
      !make_tmap_2d_bf16(&tdo, a.dO, (uint64_t)a.Hq * DH, (uint64_t)(a.B * a.Tq), (uint64_t)a.Hq * DH * 2, 64, TB2) ||
      !make_tmap_2d_bf16(&tkm, a.Mmax > 0 ? a.Kmem : a.Kloc, (uint64_t)a.Hkv * DH,
                         (uint64_t)(a.Mmax > 0 ? mrows : a.B * a.Lloc), rowkv, 64, 128) ||
      !make_tmap_2d_bf16(&tvm, a.Mmax > 0 ? a.Vmem : a.Vloc, (uint64_t)a.Hkv * DH,
                         (uint64_t)(a.Mmax > 0 ? mrows : a.B * a.Lloc), rowkv, 64, 128) ||
      !make_tmap_2d_bf16(&tkl, a.Kloc, (uint64_t)a.Hkv * DH, (uint64_t)(a.B * a.Lloc), rowkv, 64, 128) ||
      !make_tmap_2d_bf16(&tvl, a.Vloc, (uint64_t)a.Hkv * DH, (uint64_t)(a.B * a.Lloc), rowkv, 64, 128))
    return cudaErrorInvalidValue;
  DkvParams p;
  p.mem_len = a.mem_len;
  p.err_flag = a.err_flag;
  p.lse = a.lse;
  p.Drow = a.Drow;
  p.dKm = a.dKmem;
  p.dVm = a.dVmem;
  p.dKl = a.dKloc;
  p.dVl = a.dVloc;
  p.Tq = a.Tq;
  p.Lloc = a.Lloc;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.Mmax = a.Mmax;
  p.G = G;
  p.TB2 = TB2;
  p.n_qstep = (a.Tq + TB2 - 1) / TB2;
  p.n_mem_tiles = (a.Mmax + 127) / 128;
  p.chunk = pl.chunk;
  p.max_chunks = pl.max_chunks;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  cudaError_t e = cudaFuncSetAttribute(attn_dkv_tc_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  const int tiles = p.n_mem_tiles + (a.Lloc + 127) / 128;
  count_launch();
  attn_dkv_tc_kernel<DH><<<dim3((unsigned)(tiles * pl.max_chunks), (unsigned)a.Hkv, (unsigned)a.B), kDkvThreads,
                           L::kSmem, s>>>(tq, tdo, tkm, tvm, tkl, tvl, p);
  return cudaGetLastError();
}

// dQ on the tensor cores for the shapes the forward's tensor-core kernel takes
// (bf16, d = 128, a GQA group dividing 128 rows into blocks of >= 8 tokens).
cudaError_t launch_attn_dq_tc(msa_dtype dt, const AttnBwdArgs& a, cudaStream_t s, bool* handled) {
  *handled = false;
  if (dt != MSA_BF16 || a.d != 128) return cudaSuccess;
  const int G = a.Hq / a.Hkv;
  if (G < 1 || 128 % G != 0 || 128 / G < 8 || a.B > 65535 || a.Hkv > 65535) return cudaSuccess;
  constexpr int DH = 128;
  using L = DqLayout<DH>;
  const int TB = kRows / G;
  CUtensorMap tq, tdo, tkm, tvm, tkl, tvl;
  const uint64_t rowkv = (uint64_t)a.Hkv * DH * 2;
  const int64_t mrows = a.B * (int64_t)(a.Mmax > 0 ? a.Mmax : 1);
  if (!make_tmap_2d_bf16(&tq, a.Q, (uint64_t)a.Hq * DH, (uint64_t)(a.B * a.Tq), (uint64_t)a.Hq * DH * 2, 64, TB) ||
      !make_tmap_2d_bf16(&tdo, a.dO, (uint64_t)a.Hq * DH, (uint64_t)(a.B * a.Tq), (uint64_t)a.Hq * DH * 2, 64, TB) ||
      !make_tmap_2d_bf16(&tkm, a.Mmax > 0 ? a.Kmem : a.Kloc, (uint64_t)a.Hkv * DH,
                         (uint64_t)(a.Mmax > 0 ? mrows : a.B * a.Lloc), rowkv, 64, kKS) ||
      !make_tmap_2d_bf16(&tvm, a.Mmax > 0 ? a.Vmem : a.Vloc, (uint64_t)a.Hkv * DH,
                         (uint64_t)(a.Mmax > 0 ? mrows : a.B * a.Lloc), rowkv, 64, kKS) ||
      !make_tmap_2d_bf16(&tkl, a.Kloc, (uint64_t)a.Hkv * DH, (uint64_t)(a.B * a.Lloc), rowkv, 64, kKS) ||
      !make_tmap_2d_bf16(&tvl, a.Vloc, (uint64_t)a.Hkv * DH, (uint64_t)(a.B * a.Lloc), rowkv, 64, kKS))
    return cudaErrorInvalidValue;
  DqParams p;
  p.mem_len = a.mem_len;
  p.err_flag = a.err_flag;
  p.lse = a.lse;
  p.Drow = a.Drow;
  p.dQ = a.dQ;
  p.Tq = a.Tq;
  p.Lloc = a.Lloc;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.Mmax = a.Mmax;
  p.G = G;
  p.TB = TB;
  p.n_qblk = (a.Tq + TB - 1) / TB;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  cudaError_t e = cudaFuncSetAttribute(attn_dq_tc_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  *handled = true;
  count_launch();
  attn_dq_tc_kernel<DH><<<dim3((unsigned)p.n_qblk, (unsigned)a.Hkv, (unsigned)a.B), kDqThreads, L::kSmem, s>>>(
      tq, tdo, tkm, tvm, tkl, tvl, p);
  return cudaGetLastError();
}

}  // namespace msa
