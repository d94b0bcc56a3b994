// Step 5 of the MSA memory path on the 5th-generation tensor cores: softmax
// attention of the query tokens over [selected memory rows ++ causal local rows]
// ("MSA x Qwen3.5" model card, "Architecture summary"; "MSA: Memory Sparse
// Attention" README, "Architecture").
//
// Flash-style forward, one CTA per (query block, KV head, batch row):
//   * the CTA's 128 rows are the GQA group's G q-heads x (128 / G) tokens, so one
//     K/V tile serves every head of the group;
//   * key tiles of 128 rows: first the memory rows (all visible; rows past
//     mem_len are masked), then the local rows up to the block's last causal
//     position (bottom-right aligned: token i sits at Lloc - Tq + i);
//   * S = Q K^T by tcgen05.mma into one of two TMEM buffers (the tensor core
//     computes S_{j+1} while the softmax warps work on S_j); P = exp2(S - m)
//     is rounded to bf16 and written back over its own S tile in TMEM (two
//     values per 32-bit column, one row per lane), and O += P V takes P as the
//     MMA's A operand straight from tensor memory and V MN-major from its TMA
//     tile.  The tensor core runs its MMAs in issue order, so S_{j+2} (issued
//     after PV_j) never overwrites P_j before PV_j has read it;
//   * K and V tiles have separate three-deep stages: K_j is released when S_j
//     is done and V_j when PV_j is, which keeps three loads in flight against
//     the latency of a TMA tile;
//   * the running max is only moved (and O rescaled in TMEM) when it grows by
//     more than 2^8, so most tiles skip the rescale; the final 1/l and the
//     log-sum-exp use the same max, which keeps the result exact;
//   * the softmax warps are the critical path (one warp per SM sub-partition,
//     bound by instruction issue; the two that share a sub-partition with the
//     TMA and MMA warps finish last): the row max runs as eight independent
//     chains of three-input maxima, the scaled arguments and row sums use
//     packed f32x2 math, and the MMA warp reuses its operand descriptors.
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2..5 softmax / correction / output (one row per thread).
// Every wait is bounded and ends the CTA with MSA_FLAG_TIMEOUT on expiry.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace msa {
namespace {

using namespace sm100;

constexpr int kRows = 128;   // MMA M: query rows per CTA
constexpr int kKeys = 128;   // keys per tile
constexpr int kThreads = 192;
constexpr uint32_t kWaitPolls = 1u << 24;
constexpr float kRescaleLog2 = 8.0f;  // move the running max only when it grows by more than this
constexpr int kKV = 3;                // K and V stages

struct AttnTcParams {
  const int32_t* mem_len;
  int32_t* err_flag;
  __nv_bfloat16* O;
  float* lse;
  int Tq, Lloc, Hq, Hkv, Mmax, G, TB, n_qblk;
  float scale_log2;  // softmax scale * log2(e)
};

template <int DH>
struct ALayout {
  static constexpr int kBoxes = DH / 64;
  static constexpr int kQ = kRows * DH * 2;
  static constexpr int kK = kKeys * DH * 2;  // one K (or V) tile
  static constexpr int kBar = 8 * 24;
  static constexpr int kSmem = 1024 + kQ + 2 * kKV * kK + kBar;  // Q, K[kKV], V[kKV]
  static constexpr uint32_t kTmemCols = 512;  // S0, S1 (128 each), O (DH)
  static_assert(kSmem <= 232448, "shared memory of one CTA");
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic: one instruction for two values).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// max of three (exact, like any max; no NaN reaches it)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKm,
               const __grid_constant__ CUtensorMap tmVm, const __grid_constant__ CUtensorMap tmKl,
               const __grid_constant__ CUtensorMap tmVl, AttnTcParams p) {
  using L = ALayout<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Qs = smem;
  uint8_t* Ks = Qs + L::kQ;          // [kKV] K tiles
  uint8_t* Vs = Ks + kKV * L::kK;    // [kKV] V tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(Vs + kKV * L::kK);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;             // [kKV] TMA -> MMA
  uint64_t* k_empty = k_full + kKV;        // [kKV] S MMA done -> TMA
  uint64_t* v_full = k_empty + kKV;        // [kKV]
  uint64_t* v_empty = v_full + kKV;        // [kKV] PV MMA done -> TMA
  uint64_t* s_full = v_empty + kKV;        // [2] S MMA done -> softmax
  uint64_t* p_full = s_full + 2;           // [2] P written over S -> MMA
  uint64_t* p_free = p_full + 2;           // [2] PV MMA done -> softmax (O up to date)
  uint64_t* drain = p_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // longest blocks first: block index 0 takes the last query block
  const int qb = p.n_qblk - 1 - (int)blockIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int t0 = qb * p.TB;
  const int tlast = min(t0 + p.TB, p.Tq) - 1;
  int M = __ldg(p.mem_len + b);
  if (M < 0 || M > p.Mmax) {
    if (threadIdx.x == 0 && qb == 0 && g == 0) raise_flag(p.err_flag, MSA_FLAG_INDEX_OOB);
    M = M < 0 ? 0 : p.Mmax;
  }
  const int NM = (M + kKeys - 1) / kKeys;                       // memory tiles
  const int pos_last = p.Lloc - p.Tq + tlast;
  const int T = NM + (pos_last + kKeys) / kKeys;                 // + local tiles up to pos_last

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kKV; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&p_free[i], 1);
    }
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
  const uint32_t tS0 = tmem, tO = tmem + 2 * kKeys;
  bool timed_out = false;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // K and V tiles have their own stages: K_j is free once S_j is done, V_j
    // once PV_j is, and the tensor core runs S_{j+1} before PV_j, so the loads
    // go K0, K1, K2, V0, K3, V1, K4, ... in the order their stages free up.
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      mbar_arrive_expect_tx(q_full, L::kQ);
      for (int hh = 0; hh < p.G; ++hh)
#pragma unroll
        for (int dc = 0; dc < L::kBoxes; ++dc)
          tma_load_2d(Qs + dc * (kRows * 128) + hh * p.TB * 128, &tmQ, (g * p.G + hh) * DH + dc * 64,
                      b * p.Tq + t0, q_full);
      auto load = [&](int j, bool is_v) -> bool {
        const int st = j % kKV;
        uint64_t* empty = is_v ? &v_empty[st] : &k_empty[st];
        uint64_t* full = is_v ? &v_full[st] : &k_full[st];
        if (!mbar_wait(empty, ((j / kKV) & 1) ^ 1, kWaitPolls)) return false;
        uint8_t* dst = (is_v ? Vs : Ks) + st * L::kK;
        mbar_arrive_expect_tx(full, L::kK);
        const bool mem = j < NM;
        const CUtensorMap* map = is_v ? (mem ? &tmVm : &tmVl) : (mem ? &tmKm : &tmKl);
        const int y = mem ? b * p.Mmax + j * kKeys : b * p.Lloc + (j - NM) * kKeys;
#pragma unroll
        for (int dc = 0; dc < L::kBoxes; ++dc) tma_load_2d(dst + dc * (kKeys * 128), map, g * DH + dc * 64, y, full);
        return true;
      };
      int nk = 0, nv = 0;
      bool ok = true;
      while (ok && nk < kKV && nk < T) {
        if (!(ok = load(nk, false))) break;
        ++nk;
      }
      for (int j = 0; ok && j < T; ++j) {
        if (!(ok = load(j, true))) break;
        ++nv;
        if (nk < T) {
          if (!(ok = load(nk, false))) break;
          ++nk;
        }
      }
      if (!ok) timed_out = true;
      // drain the copies this thread issued
      if (!mbar_wait(q_full, 0, kWaitPolls)) timed_out = true;
      for (int st = 0; st < kKV; ++st) {
        // the last fill of stage st is fill (n - 1 - st) / kKV of it
        if (st < nk && !mbar_wait(&k_full[st], ((nk - 1 - st) / kKV) & 1, kWaitPolls)) timed_out = true;
        if (st < nv && !mbar_wait(&v_full[st], ((nv - 1 - st) / kKV) & 1, kWaitPolls)) timed_out = true;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kRows, kKeys);
      constexpr uint32_t idO = idesc_bf16_f32(kRows, DH, /*b_mn_major=*/true);
      // descriptors of the operand bases; a k-step adds its byte offset / 16 to
      // the 14-bit start-address field (shared addresses stay below 256 KB, so
      // the field never carries)
      const uint64_t dq = desc_k_sw128(smem_u32(Qs));
      const uint64_t dk0 = desc_k_sw128(smem_u32(Ks)), dv0 = desc_mn_sw128(smem_u32(Vs), kKeys * 128);
      // S_j goes to TMEM buffer j & 1, which holds P_{j-2} until PV_{j-2} has
      // read it; PV_{j-2} was issued earlier, and the MMAs run in issue order.
      auto issue_S = [&](int j) -> bool {
        const int ks = j % kKV;
        if (!mbar_wait(&k_full[ks], (j / kKV) & 1, kWaitPolls)) return false;
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)((ks * L::kK) >> 4);
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const int box = k >> 2, kk = k & 3;
          mma_bf16_ss(tS0 + (j & 1) * kKeys, dq + (uint64_t)((box * kRows * 128 + kk * 32) >> 4),
                      dk + (uint64_t)((box * kKeys * 128 + kk * 32) >> 4), idS, k > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[j & 1]);
        mma_commit(&k_empty[ks]);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, kWaitPolls) && issue_S(0);
      for (int j = 0; ok && j < T; ++j) {
        const int st = j & 1, vs = j % kKV;
        if (j + 1 < T && !issue_S(j + 1)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&p_full[st], (j >> 1) & 1, kWaitPolls) || !mbar_wait(&v_full[vs], (j / kKV) & 1, kWaitPolls)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t dv = dv0 + (uint64_t)((vs * L::kK) >> 4);
        // A = P_j from TMEM: 16 keys of bf16 per step are 8 columns
#pragma unroll
        for (int k = 0; k < kKeys / 16; ++k)
          mma_bf16_ts(tO, tS0 + st * kKeys + k * 8, dv + (uint64_t)((k * 16 * 128) >> 4), idO,
                      (j > 0 || k > 0) ? 1u : 0u);
        mma_commit(&p_free[st]);
        mma_commit(&v_empty[vs]);
      }
      if (!ok) timed_out = true;
      mma_commit(drain);
      if (!mbar_wait(drain, 0, kWaitPolls)) timed_out = true;
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int q = warp & 3;
    const int r = q * 32 + lane;                      // this thread's row (TMEM lane)
    const int hh = r / p.TB, tl = r - hh * p.TB;
    const int t = t0 + tl;
    const int pos = p.Lloc - p.Tq + t;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;  // running max in the scaled log2 domain
    for (int j = 0; j < T; ++j) {
      const int st = j & 1;
      // waits are decided warp-wide so the warp-collective tcgen05 ops are never split
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[st], (j >> 1) & 1, kWaitPolls))) {
        timed_out = true;
        break;
      }
      tc_fence_after();
      float s[kKeys];
#pragma unroll
      for (int c = 0; c < kKeys; c += 16) tmem_ld16(tmem + lane_off + st * kKeys + c, *reinterpret_cast<float(*)[16]>(&s[c]));
      tmem_ld_wait();
      // keys [0, lim) of this tile are visible to this row; most tiles are whole
      const bool memt = j < NM;
      const int base = memt ? j * kKeys : (j - NM) * kKeys;
      const int lim = memt ? M - base : pos - base + 1;
      const bool whole = __all_sync(0xffffffffu, lim >= kKeys);
      if (!whole) {
#pragma unroll
        for (int c = 0; c < kKeys; ++c) s[c] = c < lim ? s[c] : -INFINITY;
      }
      // eight independent chains of three-input maxima (max is exact in any order)
      static_assert(kKeys == 128, "the chains cover 128 keys");
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = fmax3(s[i], s[i + 8], s[i + 16]);
#pragma unroll
      for (int c = 24; c < 120; c += 16)
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmax3(m8[i], s[c + i], s[c + 8 + i]);
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = fmaxf(m8[i], s[120 + i]);
      const float mx = fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
      // move the max (and rescale O) only when it grows by more than 2^8
      const float mt = mx * sl2;
      const bool first = m_run == -INFINITY;
      const bool grow = mt > m_run + kRescaleLog2;
      float corr = 1.f;
      if (grow) {
        corr = first ? 0.f : fast_exp2(m_run - mt);
        m_run = mt;
      }
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // O must hold every earlier PV before it is rescaled
        const int jp = j - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&p_free[jp & 1], (jp >> 1) & 1, kWaitPolls))) {
          timed_out = true;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < DH; c += 16) {
          float o[16];
          tmem_ld16(tO + lane_off + c, o);
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(o[i] * corr);
          tmem_st16(tO + lane_off + c, w);
        }
        tmem_st_wait();
      }
      l_run *= corr;
      const float nm = -m_run;
      // P_j over S_j: 32 keys (16 columns of bf16 pairs) per store; the scaled arguments and the row
      // sums in packed pairs (one f32x2 instruction for two keys)
      const uint64_t sl2x2 = f2_pack(sl2, sl2), nmx2 = f2_pack(nm, nm);
      uint64_t lsa2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
      for (int c0 = 0; c0 < kKeys; c0 += 32) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[c0 + 2 * i], s[c0 + 2 * i + 1]), sl2x2, nmx2), x0, x1);
          const float e0 = fast_exp2(x0), e1 = fast_exp2(x1);
          lsa2[i & 1] = f2_add(lsa2[i & 1], f2_pack(e0, e1));
          w[i] = pack_bf16x2(e0, e1);
        }
        tmem_st16(tmem + lane_off + st * kKeys + c0 / 2, w);
      }
      float lsa[4];
      f2_unpack(lsa2[0], lsa[0], lsa[1]);
      f2_unpack(lsa2[1], lsa[2], lsa[3]);
      l_run += (lsa[0] + lsa[1]) + (lsa[2] + lsa[3]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[st]);
    }
    // output: O / l, lse = (m + log2 l) ln 2
    const int jl = T - 1;
    if (!timed_out && __all_sync(0xffffffffu, mbar_wait(&p_free[jl & 1], (jl >> 1) & 1, kWaitPolls))) {
      tc_fence_after();
      const float inv = 1.f / l_run;
      const bool rvalid = t < p.Tq;
      __nv_bfloat16* orow = p.O + (((int64_t)b * p.Tq + t) * p.Hq + g * p.G + hh) * DH;
#pragma unroll
      for (int c = 0; c < DH; c += 16) {
        float o[16];
        tmem_ld16(tO + lane_off + c, o);
        tmem_ld_wait();
        if (rvalid) {
          uint4 w0 = make_uint4(pack_bf16x2(o[0] * inv, o[1] * inv), pack_bf16x2(o[2] * inv, o[3] * inv),
                                pack_bf16x2(o[4] * inv, o[5] * inv), pack_bf16x2(o[6] * inv, o[7] * inv));
          uint4 w1 = make_uint4(pack_bf16x2(o[8] * inv, o[9] * inv), pack_bf16x2(o[10] * inv, o[11] * inv),
                                pack_bf16x2(o[12] * inv, o[13] * inv), pack_bf16x2(o[14] * inv, o[15] * inv));
          *reinterpret_cast<uint4*>(orow + c) = w0;
          *reinterpret_cast<uint4*>(orow + c + 8) = w1;
        }
      }
      if (rvalid && p.lse)
        p.lse[((int64_t)b * p.Hq + g * p.G + hh) * p.Tq + t] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
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

template <int DH>
cudaError_t launch_dh(const AttnArgs& a, cudaStream_t s) {
  using L = ALayout<DH>;
  const int G = a.Hq / a.Hkv, TB = kRows / G;
  CUtensorMap tq, tkm, tvm, tkl, tvl;
  const uint64_t rowkv = (uint64_t)a.Hkv * DH * 2;
  const int64_t mrows = a.B * (int64_t)(a.Mmax > 0 ? a.Mmax : 1);
  if (!make_tmap_2d_bf16(&tq, a.Q, (uint64_t)a.Hq * DH, (uint64_t)(a.B * a.Tq), (uint64_t)a.Hq * DH * 2, 64, TB) ||
      !make_tmap_2d_bf16(&tkm, a.Mmax > 0 ? a.Kmem : a.Kloc, (uint64_t)a.Hkv * DH, (uint64_t)(a.Mmax > 0 ? mrows : a.B * a.Lloc), rowkv, 64, kKeys) ||
      !make_tmap_2d_bf16(&tvm, a.Mmax > 0 ? a.Vmem : a.Vloc, (uint64_t)a.Hkv * DH, (uint64_t)(a.Mmax > 0 ? mrows : a.B * a.Lloc), rowkv, 64, kKeys) ||
      !make_tmap_2d_bf16(&tkl, a.Kloc, (uint64_t)a.Hkv * DH, (uint64_t)(a.B * a.Lloc), rowkv, 64, kKeys) ||
      !make_tmap_2d_bf16(&tvl, a.Vloc, (uint64_t)a.Hkv * DH, (uint64_t)(a.B * a.Lloc), rowkv, 64, kKeys))
    return cudaErrorInvalidValue;
  AttnTcParams p;
  p.mem_len = a.mem_len;
  p.err_flag = a.err_flag;
  p.O = reinterpret_cast<__nv_bfloat16*>(a.O);
  p.lse = a.lse;
  p.Tq = a.Tq;
  p.Lloc = a.Lloc;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.Mmax = a.Mmax;
  p.G = G;
  p.TB = TB;
  p.n_qblk = (a.Tq + TB - 1) / TB;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)p.n_qblk, (unsigned)a.Hkv, (unsigned)a.B);
  count_launch();
  attn_tc_kernel<DH><<<grid, kThreads, L::kSmem, s>>>(tq, tkm, tvm, tkl, tvl, p);
  return cudaGetLastError();
}

}  // namespace

// Shapes the tensor-core kernel takes: bf16, d = 128, dense memory rows, a GQA
// group that divides the 128 rows into blocks of at least 8 tokens, and enough
// query tokens to fill most of a block.
cudaError_t launch_attn_tc(msa_dtype dt, const AttnArgs& a, cudaStream_t s, bool* handled) {
  *handled = false;
  if (dt != MSA_BF16 || a.d != 128) return cudaSuccess;
  const int G = a.Hq / a.Hkv;
  if (G < 1 || 128 % G != 0 || 128 / G < 8) return cudaSuccess;
  if (a.Tq < 128 / G / 2 && a.Tq < 16) return cudaSuccess;
  if (a.B > 65535 || a.Hkv > 65535) return cudaSuccess;
  *handled = true;
  return launch_dh<128>(a, s);
}

}  // namespace msa
