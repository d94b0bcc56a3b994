// Step 5 of the MSA memory path on the 5th-generation tensor cores: softmax
// attention of the query tokens over [selected memory rows ++ causal local rows]
// ("MSA x Qwen3.5" model card, "Architecture summary"; "MSA: Memory Sparse
// Attention" README, "Architecture").
//
// Flash-style forward, one CTA per (query block, KV head, batch row):
//   * the CTA's 128 rows are the GQA group's G q-heads x (128 / G) tokens, so one
//     K/V tile serves every head of the group;
//   * key tiles of 128 rows: the local rows up to the block's last causal
//     position (bottom-right aligned: token i sits at Lloc - Tq + i), then the
//     memory rows (all visible; rows past mem_len are masked);
//   * S = Q K^T by tcgen05.mma into one of two TMEM buffers (the tensor core
//     computes S_{j+1} while the softmax warps work on S_j); P = exp2(S - m)
//     is rounded to bf16 and written back over its own S tile in TMEM (two
//     values per 32-bit column, one row per lane), and O += P V takes P as the
//     MMA's A operand straight from tensor memory and V MN-major from its TMA
//     tile.  S and PV have their own issuing threads: PV_j waits only for P_j,
//     and S_{j+2} waits for PV_j's commit before it overwrites P_j's buffer;
//   * key tile j's K and V share one of three stages and one barrier (one
//     wait per tile for both operands; separate K and V barriers made the
//     dense-memory kernel 2.4% slower); the stage is released when PV_j is done;
//   * a tile's MMAs (S and PV, 128 x 128 x 128 each) run at the tensor core's
//     full rate in isolation (~513 cycles each, B K-major or MN-major; a
//     clock64 probe of back-to-back MMAs), but the issuing thread cannot queue
//     ahead of them: issuing a group of 8 blocks about as long as it runs, and
//     each hand-off through a barrier costs a few hundred cycles.  Inside this
//     kernel PV's MMAs enter every ~79 cycles and S's every ~65; with one
//     issuer its chain per tile (issue S_{j+1}, wait for P_j, issue PV_j, wait
//     for K_{j+2}) was ~2,000 cycles, so S and PV now have one issuer each
//     (1% faster); the softmax warps' chain (S load, row max, exponentials,
//     P stores: ~1,975 cycles a tile) now paces the tile, and both issuers
//     idle about half of it.  Tried and slower: CTA pairs (cta_group::2,
//     M = 256, each CTA half of every K and V tile), P in its own TMEM columns
//     so that PV_j goes before S_{j+2}, two softmax warpgroups splitting the
//     keys;
//   * the running max is only moved (and O rescaled in TMEM) when it grows by
//     more than 2^8, so most tiles skip the rescale; the final 1/l and the
//     log-sum-exp use the same max, which keeps the result exact;
//   * the softmax warps (one per SM sub-partition): the row max runs as eight
//     independent chains of three-input maxima, the scaled arguments and row
//     sums use packed f32x2 math, six of every sixteen key pairs take a
//     polynomial 2^x on the FMA pipe instead of the transcendental unit (2-3%
//     faster than none; eight of sixteen was no better), and the MMA warps
//     reuse their operand descriptors.
// Warp roles (224 threads): warp 0 TMA producer, warp 1 TMEM owner + S MMA
// issuer, warps 2..5 softmax / correction / output (one row per thread),
// warp 6 PV MMA issuer.
// Every wait is bounded and ends the CTA with MSA_FLAG_TIMEOUT on expiry.
#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace msa {
namespace {

using namespace sm100;

constexpr int kRows = 128;   // MMA M: query rows per CTA
constexpr int kKeys = 128;   // keys per tile
constexpr int kThreads = 224;  // producer, S issuer, four softmax warps, PV issuer
constexpr uint32_t kWaitPolls = 1u << 24;
constexpr float kRescaleLog2 = 8.0f;  // move the running max only when it grows by more than this
constexpr int kKV = 3;                // K + V stages

struct AttnTcParams {
  const int32_t* mem_len;
  // index-driven memory rows (null seg_row: dense Kmem / Vmem): segment s of the
  // query starts at bank row seg_row[b * Smax + s] and holds seg_cnt[...] rows
  const int32_t* seg_row;
  const uint8_t* seg_cnt;
  const int32_t* nseg;
  int Smax;
  int32_t* err_flag;
  __nv_bfloat16* O;
  float* lse;
  int B, Tq, Lloc, Hq, Hkv, Mmax, G, TB, n_qblk;
  float scale_log2;  // softmax scale * log2(e)
  // polls of each wait that paces the pipeline (a barrier the next step needs);
  // the waits that drain this CTA's own copies and MMAs before it exits always
  // poll kWaitPolls times, so a wait that runs out still ends the CTA cleanly
  uint32_t polls;
};

template <int DH>
struct ALayout {
  static constexpr int kBoxes = DH / 64;
  static constexpr int kQ = kRows * DH * 2;
  static constexpr int kK = kKeys * DH * 2;  // one K (or V) tile
  static constexpr int kBar = 8 * 24;
  static constexpr int kSmem = 1024 + kQ + 2 * kKV * kK + kBar;  // Q, K[kKV], V[kKV]
  static constexpr uint32_t kTmemCols = 512;  // S0, S1 (128 each), O (DH), Q (DH / 2)
  static_assert(2 * kKeys + DH + DH / 2 <= (int)kTmemCols, "tensor memory columns");
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

// 2^x for a pair of arguments on the FMA and integer pipes, leaving the
// transcendental unit (whose ex2 throughput bounds the softmax) to the other
// keys: x = j + f with j = round(x) (read from the mantissa of x + 1.5 * 2^23)
// and f in [-1/2, 1/2]; 2^f by a cubic whose coefficients are a weighted
// least-squares fit of 2^f on [-1/2, 1/2] at Chebyshev nodes refined by Lawson
// iterations toward equal relative error (max relative error 7.5e-5, far below
// the bf16 rounding of P); 2^j is added to the exponent field.  Arguments below
// -126 are clamped there (weights below 2^-126 instead of 0; masked keys give
// 2^-126 * 2^f, which vanishes in the bf16 P and in the row sum's fp32).
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& e0, float& e1) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const uint64_t x = f2_pack(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
  const uint64_t t = f2_add(x, f2_pack(kMagic, kMagic));         // round(x) in the low mantissa bits
  const uint64_t jf = f2_add(t, f2_pack(-kMagic, -kMagic));      // round(x) as a float
  const uint64_t f = f2_fma(jf, f2_pack(-1.0f, -1.0f), x);        // x - round(x)
  uint64_t q = f2_fma(f, f2_pack(0.0551716648f, 0.0551716648f), f2_pack(0.2426111251f, 0.2426111251f));
  q = f2_fma(q, f, f2_pack(0.6932609677f, 0.6932609677f));
  q = f2_fma(q, f, f2_pack(0.9999280572f, 0.9999280572f));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  // the low bits of t hold round(x); shifted by 23 they add it to the exponent
  e0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  e1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// Of each 16 key pairs of a 32-key store, this many take exp2_poly2 (spread
// evenly); the rest take the transcendental unit's ex2.
constexpr int kPolyPairs = 6;
__host__ __device__ constexpr bool poly_pair(int i) { return (i * kPolyPairs) / 16 != ((i + 1) * kPolyPairs) / 16; }

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
  uint8_t* Vs = Ks + kKV * L::kK;    // [kKV] V tiles (stage st holds K_j and V_j of one key tile j)
  uint64_t* bars = reinterpret_cast<uint64_t*>(Vs + kKV * L::kK);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;            // [kKV] K and V of a key tile landed -> MMA
  uint64_t* kv_empty = kv_full + kKV;      // [kKV] PV MMA done with the stage -> TMA
  uint64_t* s_full = kv_empty + kKV;       // [2] S MMA done -> softmax
  uint64_t* p_full = s_full + 2;           // [2] P written over S -> MMA
  uint64_t* p_free = p_full + 2;           // [2] PV MMA done -> softmax (O up to date)
  uint64_t* drain = p_free + 2;
  uint64_t* q_tmem = drain + 1;            // Q copied into tensor memory (softmax threads) -> MMA
  uint64_t* drain_pv = q_tmem + 1;         // the PV issuer's own drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_pv + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // longest blocks first: block index 0 takes the last query block
  const int qb = p.n_qblk - 1 - (int)blockIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int t0 = qb * p.TB;
  const int tlast = min(t0 + p.TB, p.Tq) - 1;
  const bool bank = p.seg_row != nullptr;
  constexpr int kSegs = kKeys / kSegRows;  // segments per memory tile

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kKV; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(drain, 1);
    mbar_init(q_tmem, 128);
    mbar_init(drain_pv, 1);
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
  // TMEM columns: S0, S1 (128 each), O (DH), then Q as the S MMAs' A operand (DH / 2: bf16 pairs)
  const uint32_t tS0 = tmem, tO = tmem + 2 * kKeys, tQ = tmem + 2 * kKeys + DH;
  bool timed_out = false;
  if (warp == 0 && lane == 0) {
    // the query rows do not depend on the kernel this one may overlap
    tma_prefetch_desc(&tmQ);
    mbar_arrive_expect_tx(q_full, L::kQ);
    for (int hh = 0; hh < p.G; ++hh)
#pragma unroll
      for (int dc = 0; dc < L::kBoxes; ++dc)
        tma_load_2d(Qs + dc * (kRows * 128) + hh * p.TB * 128, &tmQ, (g * p.G + hh) * DH + dc * 64,
                    b * p.Tq + t0, q_full);
  }
  // With memory rows read from the bank, this kernel is a programmatic
  // dependent of the plan kernel: everything above overlapped it, and the plan
  // is read only after this wait (a no-op for an ordinary launch).
  pdl_wait();
  // the query's memory row count and (producer lanes) the first memory tile's run rows, both
  // loaded before either is used so their latencies overlap
  const int Mraw = bank ? __ldg(p.nseg + b) : __ldg(p.mem_len + b);
  const int seg0 = (bank && warp == 0 && lane < kSegs) ? __ldg(p.seg_row + (int64_t)b * p.Smax + lane) : 0;
  int M;
  if (bank) {
    // memory rows read in place from the bank: nseg segments of kSegRows rows
    // each, the rows past a segment's count masked like rows past mem_len
    M = min(max(Mraw, 0), p.Smax) * kSegRows;
  } else {
    M = Mraw;
    if (M < 0 || M > p.Mmax) {
      if (threadIdx.x == 0 && qb == 0 && g == 0) raise_flag(p.err_flag, MSA_FLAG_INDEX_OOB);
      M = M < 0 ? 0 : p.Mmax;
    }
  }
  const int NM = (M + kKeys - 1) / kKeys;                       // memory tiles
  const int pos_last = p.Lloc - p.Tq + tlast;
  const int NL = (pos_last + kKeys) / kKeys;                     // local tiles up to pos_last
  const int T = NL + NM;
  // Tile order: the local tiles first, then the memory tiles.  Local tile 0
  // holds a key every row sees (local row 0), so each row's running maximum is
  // finite from the first tile on; and a memory tile read from the bank (16
  // small boxes per half) is issued while earlier tiles are in flight.

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // Key tile j's K and V share stage j % kKV and one barrier, so the MMA
    // warp waits once per tile for its operands; the stage is free once PV_j
    // is done.  Lane 0 waits and arms the barrier; a memory tile read from the
    // bank is kSegs boxes of kSegRows rows per matrix, one per lane (each lands
    // on a 1 KB swizzle atom, so the tile's layout is that of one 128-row box).
    {
      auto load = [&](int j) -> bool {
        const int st = j % kKV;
        const int ok = lane == 0 ? (int)mbar_wait(&kv_empty[st], ((j / kKV) & 1) ^ 1, p.polls) : 1;
        if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
        uint8_t* dk = Ks + st * L::kK;
        uint8_t* dv = Vs + st * L::kK;
        uint64_t* full = &kv_full[st];
        if (lane == 0) mbar_arrive_expect_tx(full, 2 * L::kK);
        __syncwarp();
        const bool mem = j >= NL;
        const int jm = j - NL;  // memory tile index
        const CUtensorMap* mk = mem ? &tmKm : &tmKl;
        const CUtensorMap* mv = mem ? &tmVm : &tmVl;
        if (mem && bank) {
          if (lane < kSegs) {
            const int y = jm == 0 ? seg0 : __ldg(p.seg_row + (int64_t)b * p.Smax + jm * kSegs + lane);
#pragma unroll
            for (int dc = 0; dc < L::kBoxes; ++dc) {
              tma_load_2d(dk + dc * (kKeys * 128) + lane * (kSegRows * 128), mk, g * DH + dc * 64, y, full);
              tma_load_2d(dv + dc * (kKeys * 128) + lane * (kSegRows * 128), mv, g * DH + dc * 64, y, full);
            }
          }
        } else if (lane == 0) {
          const int y = mem ? b * p.Mmax + jm * kKeys : b * p.Lloc + j * kKeys;
#pragma unroll
          for (int dc = 0; dc < L::kBoxes; ++dc) {
            tma_load_2d(dk + dc * (kKeys * 128), mk, g * DH + dc * 64, y, full);
            tma_load_2d(dv + dc * (kKeys * 128), mv, g * DH + dc * 64, y, full);
          }
        }
        return true;
      };
      int n = 0;
      bool ok = true;
      for (; n < T; ++n)
        if (!(ok = load(n))) break;
      if (!ok) timed_out = true;
      // drain the copies this warp issued
      if (lane == 0) {
        if (!mbar_wait(q_full, 0, kWaitPolls)) timed_out = true;
        for (int st = 0; st < kKV; ++st) {
          // the last fill of stage st is fill (n - 1 - st) / kKV of it
          if (st < n && !mbar_wait(&kv_full[st], ((n - 1 - st) / kKV) & 1, kWaitPolls)) timed_out = true;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- S MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kRows, kKeys);
      // descriptors of the operand bases; a k-step adds its byte offset / 16 to
      // the 14-bit start-address field (shared addresses stay below 256 KB, so
      // the field never carries)
      const uint64_t dk0 = desc_k_sw128(smem_u32(Ks));
      auto issue_S = [&](int j) -> bool {
        const int ks = j % kKV;
        if (!mbar_wait(&kv_full[ks], (j / kKV) & 1, p.polls)) return false;
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)((ks * L::kK) >> 4);
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          // A = Q from TMEM (16 elements of bf16 per step are 8 columns), B = K from its tile
          const int box = k >> 2, kk = k & 3;
          mma_bf16_ts(tS0 + (j & 1) * kKeys, tQ + k * 8, dk + (uint64_t)((box * kKeys * 128 + kk * 32) >> 4), idS,
                      k > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[j & 1]);
        return true;
      };
      // the S MMAs read Q from tensor memory once the softmax threads have put it there; S_j
      // (j >= 2) goes into buffer j & 1 once PV_{j-2} has read P_{j-2} from it (PV is issued
      // by another thread, so the order comes from PV_{j-2}'s commit)
      bool ok = mbar_wait(q_tmem, 0, p.polls);
      for (int j = 0; ok && j < T; ++j) {
        if (j >= 2 && !mbar_wait(&p_free[j & 1], ((j - 2) >> 1) & 1, p.polls)) {
          ok = false;
          break;
        }
        if (!issue_S(j)) {
          ok = false;
          break;
        }
      }
      if (!ok) timed_out = true;
      mma_commit(drain);
      if (!mbar_wait(drain, 0, kWaitPolls)) timed_out = true;
    }
  } else if (warp == 6) {
    // ---------------------------------------------------------------- PV issuer
    if (lane == 0) {
      constexpr uint32_t idO = idesc_bf16_f32(kRows, DH, /*b_mn_major=*/true);
      const uint64_t dv0 = desc_mn_sw128(smem_u32(Vs), kKeys * 128);
      bool ok = true;
      for (int j = 0; ok && j < T; ++j) {
        const int st = j & 1, vs = j % kKV;
        // P_j written over S_j; V_j landed with K_j
        if (!mbar_wait(&p_full[st], (j >> 1) & 1, p.polls) || !mbar_wait(&kv_full[vs], (j / kKV) & 1, p.polls)) {
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
        mma_commit(&kv_empty[vs]);
      }
      if (!ok) timed_out = true;
      mma_commit(drain_pv);
      if (!mbar_wait(drain_pv, 0, kWaitPolls)) timed_out = true;
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
    // This row of Q into tensor memory: S = Q K^T then takes Q from TMEM and
    // reads only K from shared memory (both operands from shared memory would
    // use its whole read bandwidth while the TMA writes the next tiles).  The
    // row's 16-byte pieces sit in the 128-byte-swizzled layout of the TMA tile.
    if (!__all_sync(0xffffffffu, mbar_wait(q_full, 0, p.polls))) timed_out = true;
    if (!timed_out) {
      uint32_t w[DH / 2];
#pragma unroll
      for (int box = 0; box < DH / 64; ++box)
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const uint4 v = *reinterpret_cast<const uint4*>(Qs + box * (kRows * 128) + r * 128 + ((c8 ^ (r & 7)) << 4));
          w[box * 32 + c8 * 4 + 0] = v.x;
          w[box * 32 + c8 * 4 + 1] = v.y;
          w[box * 32 + c8 * 4 + 2] = v.z;
          w[box * 32 + c8 * 4 + 3] = v.w;
        }
#pragma unroll
      for (int c = 0; c < DH / 2; c += 16) tmem_st16(tQ + lane_off + c, *reinterpret_cast<const uint32_t(*)[16]>(&w[c]));
      tmem_st_wait();
    }
    tc_fence_before();
    mbar_arrive(q_tmem);
    float m_run = -INFINITY, l_run = 0.f;  // running max in the scaled log2 domain
    for (int j = 0; j < T; ++j) {
      const int st = j & 1;
      // a bank tile's segment counts (one byte per segment), loaded before the wait
      uint4 segc = make_uint4(0u, 0u, 0u, 0u);
      if (bank && j >= NL)
        segc = __ldg(reinterpret_cast<const uint4*>(p.seg_cnt + (int64_t)b * p.Smax + (j - NL) * kSegs));
      // waits are decided warp-wide so the warp-collective tcgen05 ops are never split
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[st], (j >> 1) & 1, p.polls))) {
        timed_out = true;
        break;
      }
      tc_fence_after();
      float s[kKeys];
#pragma unroll
      for (int c = 0; c < kKeys; c += 16) tmem_ld16(tmem + lane_off + st * kKeys + c, *reinterpret_cast<float(*)[16]>(&s[c]));
      tmem_ld_wait();
      // keys [0, lim) of this tile are visible to this row; most tiles are whole
      const bool memt = j >= NL;
      if (memt && bank) {
        // key c of the tile is row c % kSegRows of segment c / kSegRows
        static_assert(kSegs == 16 && kSegRows == 8, "four segment counts per word");
        const uint32_t full8 = 0x08080808u;
        if (!(segc.x == full8 && segc.y == full8 && segc.z == full8 && segc.w == full8)) {
          const uint32_t cw[4] = {segc.x, segc.y, segc.z, segc.w};
#pragma unroll
          for (int c = 0; c < kKeys; ++c) {
            const uint32_t n = (cw[c >> 5] >> (((c >> 3) & 3) * 8)) & 0xffu;
            s[c] = (uint32_t)(c & 7) < n ? s[c] : -INFINITY;
          }
        }
      } else {
        const int base = memt ? (j - NL) * kKeys : j * kKeys;
        const int lim = memt ? M - base : pos - base + 1;
        const bool whole = __all_sync(0xffffffffu, lim >= kKeys);
        if (!whole) {
#pragma unroll
          for (int c = 0; c < kKeys; ++c) s[c] = c < lim ? s[c] : -INFINITY;
        }
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
        if (!__all_sync(0xffffffffu, mbar_wait(&p_free[jp & 1], (jp >> 1) & 1, p.polls))) {
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
          float x0, x1, e0, e1;
          f2_unpack(f2_fma(f2_pack(s[c0 + 2 * i], s[c0 + 2 * i + 1]), sl2x2, nmx2), x0, x1);
          if (poly_pair(i)) {
            exp2_poly2(x0, x1, e0, e1);
          } else {
            e0 = fast_exp2(x0);
            e1 = fast_exp2(x1);
          }
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
    if (!timed_out && __all_sync(0xffffffffu, mbar_wait(&p_free[jl & 1], (jl >> 1) & 1, p.polls))) {
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

// Polls of the pipeline waits (negative: kWaitPolls); tests of the expiry path set it.
std::atomic<int64_t> g_test_polls{-1};

template <int DH>
cudaError_t launch_dh(const AttnArgs& a, cudaStream_t s) {
  using L = ALayout<DH>;
  const int G = a.Hq / a.Hkv, TB = kRows / G;
  CUtensorMap tq, tkm, tvm, tkl, tvl;
  const uint64_t rowkv = (uint64_t)a.Hkv * DH * 2;
  const int64_t mrows = a.B * (int64_t)(a.Mmax > 0 ? a.Mmax : 1);
  const bool bank = a.seg_row != nullptr;
  // memory maps: the bank [C, Hkv * d] in boxes of one segment, or the dense rows [B * Mmax, Hkv * d]
  const void* km = bank || a.Mmax > 0 ? a.Kmem : a.Kloc;
  const void* vm = bank || a.Mmax > 0 ? a.Vmem : a.Vloc;
  const uint64_t mr = bank ? (uint64_t)(a.C > 0 ? a.C : 1) : (uint64_t)(a.Mmax > 0 ? mrows : a.B * a.Lloc);
  const uint32_t mbox = bank ? kSegRows : kKeys;
  if (!make_tmap_2d_bf16(&tq, a.Q, (uint64_t)a.Hq * DH, (uint64_t)(a.B * a.Tq), (uint64_t)a.Hq * DH * 2, 64, TB) ||
      !make_tmap_2d_bf16(&tkm, km, (uint64_t)a.Hkv * DH, mr, rowkv, 64, mbox) ||
      !make_tmap_2d_bf16(&tvm, vm, (uint64_t)a.Hkv * DH, mr, rowkv, 64, mbox) ||
      !make_tmap_2d_bf16(&tkl, a.Kloc, (uint64_t)a.Hkv * DH, (uint64_t)(a.B * a.Lloc), rowkv, 64, kKeys) ||
      !make_tmap_2d_bf16(&tvl, a.Vloc, (uint64_t)a.Hkv * DH, (uint64_t)(a.B * a.Lloc), rowkv, 64, kKeys))
    return cudaErrorInvalidValue;
  AttnTcParams p;
  p.mem_len = a.mem_len;
  p.seg_row = a.seg_row;
  p.seg_cnt = a.seg_cnt;
  p.nseg = a.nseg;
  p.Smax = a.Smax;
  p.err_flag = a.err_flag;
  p.O = reinterpret_cast<__nv_bfloat16*>(a.O);
  p.lse = a.lse;
  p.B = (int)a.B;
  p.Tq = a.Tq;
  p.Lloc = a.Lloc;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.Mmax = a.Mmax;
  p.G = G;
  p.TB = TB;
  p.n_qblk = (a.Tq + TB - 1) / TB;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  const int64_t tp = g_test_polls.load(std::memory_order_relaxed);
  p.polls = tp < 0 ? kWaitPolls : (uint32_t)(tp < (int64_t)kWaitPolls ? tp : kWaitPolls);
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)p.n_qblk, (unsigned)a.Hkv, (unsigned)a.B);
  count_launch();
  if (a.seg_row)  // overlaps the plan kernel just before it on the stream
    return launch_pdl(attn_tc_kernel<DH>, grid, dim3(kThreads), (size_t)L::kSmem, s, tq, tkm, tvm, tkl, tvl, p);
  attn_tc_kernel<DH><<<grid, kThreads, L::kSmem, s>>>(tq, tkm, tvm, tkl, tvl, p);
  return cudaGetLastError();
}

}  // namespace

// Shapes the tensor-core kernel takes: bf16, d = 128, dense memory rows, a GQA
// group that divides the 128 rows into blocks of at least 8 tokens, and enough
// query tokens to fill most of a block.
void attn_tc_set_test_polls(int64_t polls) { g_test_polls.store(polls, std::memory_order_relaxed); }

bool attn_tc_applies(msa_dtype dt, const AttnArgs& a) {
  if (dt != MSA_BF16 || a.d != 128) return false;
  const int G = a.Hq / a.Hkv;
  if (G < 1 || 128 % G != 0 || 128 / G < 8) return false;
  if (a.Tq < 128 / G / 2 && a.Tq < 16) return false;
  return a.B <= 65535 && a.Hkv <= 65535;
}

cudaError_t launch_attn_tc(msa_dtype dt, const AttnArgs& a, cudaStream_t s, bool* handled) {
  *handled = attn_tc_applies(dt, a);
  if (!*handled) return cudaSuccess;
  return launch_dh<128>(a, s);
}

}  // namespace msa
