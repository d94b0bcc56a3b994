// Step 5 of the MSA memory path for decoding: a few query tokens per batch row
// attending over [selected memory rows ++ the whole local KV]
// ("MSA x Qwen3.5" model card, "Architecture summary"; "MSA: Memory Sparse
// Attention" README, "Inference Pipeline" stage 3, sparse generation).
//
// Decoding reads every K and V row once and does little arithmetic per row, so
// the kernel is shaped for HBM bandwidth; the contractions still run on the
// tensor cores, with the roles of prefill swapped so that the 128 keys of a
// tile are the MMA's M (one TMEM lane each) and the R = G * Tq <= 16 query
// rows of one KV head are its N = 16:
//   S^T[key, row] = K_tile (TMA, 128-byte swizzle) x Q^T        (tcgen05.mma)
//   O^T[d, row]  += V_tile^T (MN-major, straight from the tile) x P^T
// with S^T double-buffered in TMEM and P^T in shared memory, so the tensor
// core computes the next tile while the softmax warps work on this one; the
// MMA thread polls its barriers without blocking and issues each tile's S and
// P V as soon as their inputs are ready.  Each softmax thread owns one TMEM
// lane: a key of S^T and a dimension of O^T.  Column (row) maxima are reduced
// across the 128 lanes with shuffles and shared memory; the running max moves
// only when it grows by more than 2^8 (then O^T is rescaled in TMEM).
// One CTA per SM streams an equal, contiguous share of all (batch row, KV
// head, key tile) triples; each stretch of that share inside one (batch row,
// KV head) is a segment, which leaves (max, sum, unnormalised O) per row in the
// workspace, and a second kernel merges the segments.  The softmax threads
// handle only the R real query rows (rounded up to 4, 8 or 16), and load the
// next segment's Q rows while the current one streams, into the other of two
// Q buffers.
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2..5 softmax / output.  Every wait is bounded; after the first
// expired wait the CTA stops waiting, runs its loops out without data and
// raises MSA_FLAG_TIMEOUT.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace msa {
namespace {

using namespace sm100;

constexpr int kDH = 128;
constexpr int kKeys = 128;              // keys per tile (the MMA's M)
constexpr int kMaxRows = 16;            // R = G * Tq (the MMA's N, padded to 16)
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr uint32_t kWaitPolls = 1u << 24;
constexpr uint32_t kSpinLimit = 1u << 28;  // non-blocking polls of the MMA issuer without progress
constexpr float kRescaleLog2 = 8.0f;

struct DecParams {
  const __nv_bfloat16* Q;
  const int32_t* mem_len;
  // index-driven memory rows (null seg_row: dense Kmem / Vmem): segment s of
  // batch row b starts at bank row seg_row[b * plan_smax + s] and holds
  // seg_cnt[...] rows; memory tile t holds segments [16 t, 16 t + 16)
  const int32_t* seg_row;
  const uint8_t* seg_cnt;
  int plan_smax;
  int32_t* err_flag;
  float* part;  // [B * Hkv][Smax][R][kDH + 2]: m, l, O of one segment
  int64_t B;
  int Tq, Lloc, Hq, Hkv, Mmax, G, R;
  int NM;       // memory tiles (ceil(Mmax / kKeys), or Smax / 16 from a plan); masked rows as above
  int NL;       // local tiles (ceil(Lloc / kKeys))
  int T;        // tiles per (b, g): NM + NL
  int Smax;     // partial slots per (b, g)
  int64_t Ttot, per;  // all tiles (B * Hkv * T) and tiles per CTA
  float scale_log2;
};

struct DLayout {
  static constexpr int kTile = kKeys * kDH * 2;       // one K (or V) tile, two 64-wide boxes
  static constexpr int kStage = 2 * kTile;
  static constexpr int kQ = kMaxRows * kDH * 2;       // Q rows, K-major, 128-byte swizzle (two buffers)
  static constexpr int kP = kMaxRows * kKeys * 2;     // P^T rows (query rows x keys); two buffers
  static constexpr int kRed = 3 * kMaxRows * 4 * 4;    // [2 tile parities + segment end][rows][4 warps]
  static constexpr int kSmem = 1024 + kStages * kStage + 2 * kQ + 2 * kP + kRed + 8 * 18 + 16;
  static constexpr uint32_t kTmemCols = 64;           // S0, S1, O (16 columns each)
};

// One CTA's share of the work is the contiguous range [f0, f1) of the flattened
// tile index f = (b * Hkv + g) * T + t, so every CTA streams the same number of
// tiles; a segment is the part of that range that lies in one (b, g).  The
// segment's partial result goes to slot (CTA - first CTA touching (b, g)).
struct Seg {
  int64_t bg;
  int t0, t1, slot;
};
__device__ __forceinline__ Seg seg_at(const DecParams& p, int64_t f, int64_t f1) {
  Seg s;
  s.bg = f / p.T;
  s.t0 = (int)(f - s.bg * p.T);
  s.t1 = (int)min((int64_t)p.T, (int64_t)s.t0 + (f1 - f));
  s.slot = (int)((int64_t)blockIdx.x - (s.bg * p.T) / p.per);
  return s;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void bar_softmax() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Maximum of v over the 32 lanes, in every lane (one instruction on sm_100a).
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Byte offset of element (row, col) in a K-major, 128-byte-swizzled tile whose
// rows hold 64 elements per box and `rows` rows per box.
__device__ __forceinline__ int sw128_off(int row, int col, int rows) {
  const int box = col >> 6, c = col & 63;
  return box * (rows * 128) + row * 128 + ((((c >> 3) ^ (row & 7))) << 4) + (c & 7) * 2;
}

// kR >= R is the number of query rows the softmax threads handle (4, 8 or 16);
// the MMA's N stays 16 and the columns past kR are never read.
template <int kR>
__global__ void __launch_bounds__(kThreads, 1)
attn_decode_kernel(const __grid_constant__ CUtensorMap tmKm, const __grid_constant__ CUtensorMap tmVm,
                   const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmVl, DecParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* Qs = ring + kStages * DLayout::kStage;  // two buffers, alternating by segment
  uint8_t* Ps = Qs + 2 * DLayout::kQ;
  float* red_s = reinterpret_cast<float*>(Ps + 2 * DLayout::kP);  // [3][16 rows][4 warps]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red_s) + DLayout::kRed);
  uint64_t* kv_full = bars;            // [3]
  uint64_t* kv_empty = bars + 3;       // [3]
  uint64_t* s_full = bars + 6;         // [2]
  uint64_t* s_free = bars + 8;         // [2]
  uint64_t* q_ready = bars + 10;
  uint64_t* p_full = bars + 11;        // [2] per P buffer
  uint64_t* o_done = bars + 13;        // [2] per P buffer: its P V has completed
  uint64_t* drain = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_s = reinterpret_cast<volatile int*>(bars + 17);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t f0 = (int64_t)blockIdx.x * p.per, f1 = min(f0 + p.per, p.Ttot);
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    mbar_init(q_ready, 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drain, 1);
    *abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, DLayout::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 32;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // Lane 0 waits and arms the barriers; a memory tile read from the bank is 16
    // boxes of kSegRows rows (one segment each), issued by lanes 0..15, each
    // landing on a 1 KB swizzle atom so the tile's layout is that of one box.
    const bool bank = p.seg_row != nullptr;
    uint32_t it = 0;
    bool stop = false;
    for (int64_t f = f0; f < f1 && !stop;) {
      const Seg sg = seg_at(p, f, f1);
      const int g = (int)(sg.bg % p.Hkv);
      const int64_t b = sg.bg / p.Hkv;
      for (int t = sg.t0; t < sg.t1; ++t, ++it) {
        const uint32_t st = it % kStages, round = it / kStages;
        int ok = 1;
        if (lane == 0) {
          ok = !*abort_s && mbar_wait(&kv_empty[st], (round & 1) ^ 1, kWaitPolls);
          if (!ok) *abort_s = 1;
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          stop = true;
          break;
        }
        uint8_t* Kd = ring + st * DLayout::kStage;
        uint8_t* Vd = Kd + DLayout::kTile;
        if (lane == 0) mbar_arrive_expect_tx(&kv_full[st], DLayout::kStage);
        __syncwarp();
        const bool mem = t < p.NM;
        const CUtensorMap* mk = mem ? &tmKm : &tmKl;
        const CUtensorMap* mv = mem ? &tmVm : &tmVl;
        if (mem && bank) {
          if (lane < kKeys / kSegRows) {
            const int y = __ldg(p.seg_row + b * p.plan_smax + t * (kKeys / kSegRows) + lane);
            const int so = lane * (kSegRows * 128);
            for (int dc = 0; dc < 2; ++dc) {
              tma_load_2d(Kd + dc * (kKeys * 128) + so, mk, g * kDH + dc * 64, y, &kv_full[st]);
              tma_load_2d(Vd + dc * (kKeys * 128) + so, mv, g * kDH + dc * 64, y, &kv_full[st]);
            }
          }
        } else if (lane == 0) {
          const int y = mem ? (int)(b * p.Mmax + t * kKeys) : (int)(b * p.Lloc + (t - p.NM) * kKeys);
          for (int dc = 0; dc < 2; ++dc) {
            tma_load_2d(Kd + dc * (kKeys * 128), mk, g * kDH + dc * 64, y, &kv_full[st]);
            tma_load_2d(Vd + dc * (kKeys * 128), mv, g * kDH + dc * 64, y, &kv_full[st]);
          }
        }
      }
      f += sg.t1 - sg.t0;
    }
    if (lane == 0) {
      const uint32_t fills = it;
      for (uint32_t st = 0; st < (uint32_t)kStages && st < fills; ++st) {
        const uint32_t last = (fills - 1 - st) / kStages * kStages + st;
        if (!mbar_wait(&kv_full[st], (last / kStages) & 1, kWaitPolls)) *abort_s = 1;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kKeys, kMaxRows);                              // K x Q^T
      constexpr uint32_t idO = idesc_bf16_f32(kDH, kMaxRows, /*b_mn=*/false, /*a_mn=*/true);  // V^T x P^T
      const uint32_t p0 = smem_u32(Ps);
      uint32_t it = 0, js = 0, nseg = 0;  // it: K/V tiles; js: S buffers used; nseg: segments
      for (int64_t f = f0; f < f1; ++nseg) {
        const Seg sg = seg_at(p, f, f1);
        const int T = sg.t1 - sg.t0;
        const uint32_t q0 = smem_u32(Qs + (nseg & 1) * DLayout::kQ);
        if (!*abort_s && !mbar_wait(q_ready, nseg & 1, kWaitPolls)) *abort_s = 1;
        // Issue S = K Q^T of a tile as soon as its K/V stage and an S buffer are
        // ready, and O += V^T P^T of a tile as soon as its P is: one thread polls
        // both (test_wait does not block), so a tile's P V is never held back by
        // the next tile's copy.  Tile g = it + j (over the CTA's whole range)
        // uses P buffer g & 1, phase g >> 1.
        int nS = 0, nP = 0;
        uint32_t spins = 0;
        while (nP < T && !*abort_s) {
          bool prog = false;
          if (nS < T) {
            const uint32_t g = it + nS, st = g % kStages, round = g / kStages;
            const uint32_t sb = (js + nS) & 1, use = (js + nS) >> 1;
            if (mbar_test(&kv_full[st], round & 1) && mbar_test(&s_free[sb], (use & 1) ^ 1)) {
              tc_fence_after();
              const uint32_t k0 = smem_u32(ring + st * DLayout::kStage);
#pragma unroll
              for (int k = 0; k < kDH / 16; ++k) {
                const int box = k >> 2, kk = k & 3;
                mma_bf16_ss(tS + sb * 16, desc_k_sw128(k0 + box * (kKeys * 128) + kk * 32),
                            desc_k_sw128(q0 + box * (kMaxRows * 128) + kk * 32), idS, k > 0 ? 1u : 0u);
              }
              mma_commit(&s_full[sb]);
              ++nS;
              prog = true;
            }
          }
          if (nP < nS) {
            const uint32_t g = it + nP, st = g % kStages, pb = g & 1;
            if (mbar_test(&p_full[pb], (g >> 1) & 1)) {
              tc_fence_after();
              const uint32_t v0 = smem_u32(ring + st * DLayout::kStage + DLayout::kTile);
              const uint32_t pp = p0 + pb * DLayout::kP;
#pragma unroll
              for (int k = 0; k < kKeys / 16; ++k) {
                const int box = k >> 2, kk = k & 3;
                mma_bf16_ss(tO, desc_mn_sw128(v0 + k * 16 * 128, kKeys * 128),
                            desc_k_sw128(pp + box * (kMaxRows * 128) + kk * 32), idO, (nP > 0 || k > 0) ? 1u : 0u);
              }
              mma_commit(&o_done[pb]);
              mma_commit(&kv_empty[st]);
              ++nP;
              prog = true;
            }
          }
          if (prog) spins = 0;
          else if (++spins > kSpinLimit) *abort_s = 1;
        }
        it += T;
        js += T;
        f += T;
      }
      mma_commit(drain);
      if (!mbar_wait(drain, 0, kWaitPolls)) *abort_s = 1;
    }
  } else {
    // ---------------------------------------------------------------- softmax / output
    const int q = warp & 3;
    const int r_lane = q * 32 + lane;               // this thread's TMEM lane: key of S^T, dim of O^T
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int et = tid - 64;                        // 0..127
    // Q rows of a segment into a swizzled K-major buffer: element i of R * 16
    // 16-byte pieces is row r = i / 16 (token r / G, head g * G + r % G).
    auto load_q = [&](const Seg& sg, uint4 (&v)[2]) {
      const int g = (int)(sg.bg % p.Hkv);
      const int64_t b = sg.bg / p.Hkv;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int i = et + 128 * k, r = i >> 4, c8 = (i & 15) * 8;
        v[k] = make_uint4(0, 0, 0, 0);
        if (r < p.R) {
          const int t = r / p.G, h = g * p.G + r % p.G;
          v[k] = __ldg(reinterpret_cast<const uint4*>(p.Q + ((b * p.Tq + t) * p.Hq + h) * (int64_t)kDH + c8));
        }
      }
    };
    auto store_q = [&](uint8_t* buf, const uint4 (&v)[2]) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int i = et + 128 * k, r = i >> 4, c8 = (i & 15) * 8;
        if (r < p.R) *reinterpret_cast<uint4*>(buf + sw128_off(r, c8, kMaxRows)) = v[k];
      }
    };
    // rows past R stay zero in both buffers; segment 0's rows go to buffer 0
    for (int i = et; i < 2 * kMaxRows * (kDH / 8); i += 128) {
      const int bsel = i / (kMaxRows * (kDH / 8)), r = (i >> 4) % kMaxRows, c8 = (i & 15) * 8;
      if (r >= p.R) *reinterpret_cast<uint4*>(Qs + bsel * DLayout::kQ + sw128_off(r, c8, kMaxRows)) = make_uint4(0, 0, 0, 0);
    }
    {
      uint4 v[2];
      load_q(seg_at(p, f0, f1), v);
      store_q(Qs, v);
    }
    fence_async_smem();
    tc_fence_before();
    mbar_arrive(q_ready);

    uint32_t it = 0, js = 0, nseg = 0;
    for (int64_t f = f0; f < f1; ++nseg) {
      const Seg sg = seg_at(p, f, f1);
      const int64_t b = sg.bg / p.Hkv;
      const int t0 = sg.t0;
      const int T = sg.t1 - sg.t0;
      const int64_t fn = f + T;
      // the next segment's Q rows, loaded now and stored after this segment's first tile
      uint4 qn[2];
      if (fn < f1) load_q(seg_at(p, fn, f1), qn);
      const bool bank = p.seg_row != nullptr;
      int M = bank ? 0 : __ldg(p.mem_len + b);
      if (M < 0 || M > p.Mmax) {
        if (et == 0 && sg.t0 == 0 && sg.bg % p.Hkv == 0) raise_flag(p.err_flag, MSA_FLAG_INDEX_OOB);
        M = M < 0 ? 0 : p.Mmax;
      }
      float m_run[kR], l_run[kR];
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        m_run[r] = -INFINITY;
        l_run[r] = 0.f;
      }
      for (int j = 0; j < T; ++j) {
        const int t = t0 + j;
        const uint32_t sb = (js + j) & 1, use = (js + j) >> 1;
        // a bank tile: this thread's key is row (r_lane % kSegRows) of segment 16 t + r_lane / kSegRows
        int seg_n = 0;
        if (bank && t < p.NM) seg_n = __ldg(p.seg_cnt + b * p.plan_smax + t * (kKeys / kSegRows) + (r_lane >> 3));
        if (!*abort_s && !__all_sync(0xffffffffu, mbar_wait(&s_full[sb], use & 1, kWaitPolls))) *abort_s = 1;
        tc_fence_after();
        float sc[kR];
        tmem_ld_cols<kR>(tS + sb * 16 + lane_off, sc);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s_free[sb]);
        // mask; scale into the log2 domain
        const bool mem = t < p.NM;
        const int key = (mem ? t : t - p.NM) * kKeys + r_lane;
        const bool mem_vis = bank ? (r_lane & (kSegRows - 1)) < seg_n : key < M;
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          const bool vis = r < p.R && (mem ? mem_vis : key <= p.Lloc - p.Tq + r / p.G);
          sc[r] = vis ? sc[r] * p.scale_log2 : -INFINITY;
        }
        // column maxima over the tile's 128 keys: a warp reduction per column,
        // then the four warps' maxima through shared memory.  The exchange
        // buffer alternates with the tile's parity, so one barrier per tile
        // suffices (a buffer is rewritten two tiles later, after every thread
        // has passed the barrier of the tile in between).
        float* red = red_s + ((it + j) & 1) * (kMaxRows * 4);
        float mine = -INFINITY;  // lane r < kR keeps this warp's maximum of column r
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          const float v = warp_max(sc[r]);
          mine = lane == r ? v : mine;
        }
        if (lane < kR) red[lane * 4 + q] = mine;
        bar_softmax();
        bool grow = false;
        float corr[kR];
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          const float4 w = *reinterpret_cast<const float4*>(red + r * 4);
          const float mt = fmaxf(fmaxf(w.x, w.y), fmaxf(w.z, w.w));
          corr[r] = 1.f;
          if (mt > m_run[r] + kRescaleLog2) {  // same decision in every thread
            corr[r] = m_run[r] == -INFINITY ? 0.f : fast_exp2(m_run[r] - mt);
            m_run[r] = mt;
            grow = true;
          }
        }
        float pr[kR];
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          pr[r] = sc[r] == -INFINITY ? 0.f : fast_exp2(sc[r] - m_run[r]);
          l_run[r] = l_run[r] * corr[r] + pr[r];
        }
        // P buffer g & 1 was last read by the P V of tile g - 2; O is rescaled
        // only after the P V of tile g - 1
        const uint32_t g = it + j;
        if (g >= 2 && !*abort_s &&
            !__all_sync(0xffffffffu, mbar_wait(&o_done[g & 1], ((g - 2) >> 1) & 1, kWaitPolls)))
          *abort_s = 1;
        if (j > 0 && grow && !*abort_s &&
            !__all_sync(0xffffffffu, mbar_wait(&o_done[(g - 1) & 1], ((g - 1) >> 1) & 1, kWaitPolls)))
          *abort_s = 1;
        if (j > 0 && grow) {
          tc_fence_after();
          float o[kR];
          tmem_ld_cols<kR>(tO + lane_off, o);
          tmem_ld_wait();
          uint32_t w[kR];
#pragma unroll
          for (int r = 0; r < kR; ++r) w[r] = __float_as_uint(o[r] * corr[r]);
          tmem_st_cols<kR>(tO + lane_off, w);
          tmem_st_wait();
        }
#pragma unroll
        for (int r = 0; r < kR; ++r)
          *reinterpret_cast<__nv_bfloat16*>(Ps + (g & 1) * DLayout::kP + sw128_off(r, r_lane, kMaxRows)) =
              __float2bfloat16_rn(pr[r]);
        // The other Q buffer was last read by the previous segment's S MMAs,
        // all complete before that segment's last P V.
        if (j == 0 && fn < f1) store_q(Qs + ((nseg + 1) & 1) * DLayout::kQ, qn);
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&p_full[g & 1]);
        if (j == 0 && fn < f1) mbar_arrive(q_ready);
      }
      // segment result: O^T[d = r_lane][row], the row maxima and the summed weights
      {
        const uint32_t g = it + T - 1;  // the segment's last tile
        if (!*abort_s && !__all_sync(0xffffffffu, mbar_wait(&o_done[g & 1], (g >> 1) & 1, kWaitPolls)))
          *abort_s = 1;
      }
      tc_fence_after();
      float o[kR];
      tmem_ld_cols<kR>(tO + lane_off, o);
      tmem_ld_wait();
      float* out = p.part + (size_t)(sg.bg * p.Smax + sg.slot) * p.R * (kDH + 2);
      float* red_l = red_s + 2 * (kMaxRows * 4);  // the segment's row sums, apart from the tile buffers
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        float v = l_run[r];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) red_l[r * 4 + q] = v;
        if (r < p.R) out[r * (kDH + 2) + 2 + r_lane] = o[r];
      }
      bar_softmax();
      if (et < p.R) {
        float m = -INFINITY;
#pragma unroll
        for (int r = 0; r < kR; ++r) m = r == et ? m_run[r] : m;
        out[et * (kDH + 2)] = m;
        out[et * (kDH + 2) + 1] = red_l[et * 4] + red_l[et * 4 + 1] + red_l[et * 4 + 2] + red_l[et * 4 + 3];
      }
      bar_softmax();
      tc_fence_before();
      it += T;
      js += T;
      f = fn;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, DLayout::kTmemCols);
  }
  if (tid == 0 && *abort_s) raise_flag(p.err_flag, MSA_FLAG_TIMEOUT);
}

// Merge the segments of every (b, g) row: O = sum_s 2^(m_s - m) O_s / sum_s 2^(m_s - m) l_s.
// The segments of (b, g) are those of the CTAs whose tile ranges meet its tiles.
__global__ void decode_combine_kernel(DecParams p, __nv_bfloat16* __restrict__ O, float* __restrict__ lse) {
  const int64_t bg = blockIdx.x;  // one CTA per (b, g), one warp per row
  const int g = (int)(bg % p.Hkv);
  const int64_t b = bg / p.Hkv;
  const int r = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (r >= p.R) return;
  const int ns = (int)((bg * p.T + p.T - 1) / p.per - (bg * p.T) / p.per + 1);
  const float* base = p.part + (size_t)bg * p.Smax * p.R * (kDH + 2);
  float m = -INFINITY;
  for (int s = 0; s < ns; ++s) m = fmaxf(m, base[((size_t)s * p.R + r) * (kDH + 2)]);
  float l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < ns; ++s) {
    const float* src = base + ((size_t)s * p.R + r) * (kDH + 2);
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
  int R, NM, NL, T, Smax;
  int64_t bgs, Ttot, per, grid;
};

DecodePlan plan(const AttnArgs& a) {
  DecodePlan d{};
  d.R = (a.Hq / a.Hkv) * a.Tq;
  d.NM = a.seg_row ? a.Smax / (kKeys / kSegRows) : (a.Mmax + kKeys - 1) / kKeys;
  d.NL = (a.Lloc + kKeys - 1) / kKeys;
  d.T = d.NM + d.NL;
  d.bgs = a.B * a.Hkv;
  d.Ttot = d.bgs * d.T;
  if (d.Ttot <= 0) return d;
  // one CTA per SM, each streaming an equal contiguous share of all tiles
  const int64_t g0 = d.Ttot < sm_count() ? d.Ttot : sm_count();
  d.per = (d.Ttot + g0 - 1) / g0;
  d.grid = (d.Ttot + d.per - 1) / d.per;
  // a (b, g) of T tiles meets at most (T - 1) / per + 2 consecutive ranges
  int64_t smax = (d.T - 1) / d.per + 2;
  d.Smax = (int)(smax < d.grid ? smax : d.grid);
  return d;
}

}  // namespace

bool decode_applies(msa_dtype dt, const AttnArgs& a) {
  if (dt != MSA_BF16 || a.d != kDH || a.Hq % a.Hkv) return false;
  const int R = (a.Hq / a.Hkv) * a.Tq;
  return R <= kMaxRows && a.Tq <= 4;
}

size_t decode_workspace_size_smax(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int Smax) {
  AttnArgs a{};
  a.B = B;
  a.Tq = Tq;
  a.Lloc = Lloc;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Smax = Smax;
  a.seg_row = reinterpret_cast<const int32_t*>(16);  // marks the plan layout; never dereferenced
  const DecodePlan d = plan(a);
  return sizeof(float) * (size_t)d.bgs * d.Smax * d.R * (kDH + 2);
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
  return sizeof(float) * (size_t)d.bgs * d.Smax * d.R * (kDH + 2);
}

cudaError_t launch_attn_decode(const AttnArgs& a, cudaStream_t s) {
  const DecodePlan d = plan(a);
  if (d.Ttot <= 0) return cudaSuccess;
  const size_t need = sizeof(float) * (size_t)d.bgs * d.Smax * d.R * (kDH + 2);
  if (!a.ws || a.ws_bytes < need) return cudaErrorInvalidValue;
  CUtensorMap tkm, tvm, tkl, tvl;
  const uint64_t rowkv = (uint64_t)a.Hkv * kDH * 2;
  const int64_t mrows = a.B * (int64_t)(a.Mmax > 0 ? a.Mmax : 1);
  const bool bank = a.seg_row != nullptr;
  // memory maps: the bank [C, Hkv * d] in boxes of one segment, or the dense rows [B * Mmax, Hkv * d]
  const void* km = bank || a.Mmax > 0 ? a.Kmem : a.Kloc;
  const void* vm = bank || a.Mmax > 0 ? a.Vmem : a.Vloc;
  const uint64_t mr = bank ? (uint64_t)(a.C > 0 ? a.C : 1) : (uint64_t)(a.Mmax > 0 ? mrows : a.B * a.Lloc);
  const uint32_t mbox = bank ? kSegRows : kKeys;
  if (!make_tmap_2d_bf16(&tkm, km, (uint64_t)a.Hkv * kDH, mr, rowkv, 64, mbox) ||
      !make_tmap_2d_bf16(&tvm, vm, (uint64_t)a.Hkv * kDH, mr, rowkv, 64, mbox) ||
      !make_tmap_2d_bf16(&tkl, a.Kloc, (uint64_t)a.Hkv * kDH, (uint64_t)(a.B * a.Lloc), rowkv, 64, kKeys) ||
      !make_tmap_2d_bf16(&tvl, a.Vloc, (uint64_t)a.Hkv * kDH, (uint64_t)(a.B * a.Lloc), rowkv, 64, kKeys))
    return cudaErrorInvalidValue;
  DecParams p;
  p.Q = reinterpret_cast<const __nv_bfloat16*>(a.Q);
  p.mem_len = a.mem_len;
  p.seg_row = a.seg_row;
  p.seg_cnt = a.seg_cnt;
  p.plan_smax = a.Smax;
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
  p.T = d.T;
  p.Smax = d.Smax;
  p.Ttot = d.Ttot;
  p.per = d.per;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  auto kern = d.R <= 4 ? attn_decode_kernel<4> : (d.R <= 8 ? attn_decode_kernel<8> : attn_decode_kernel<16>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DLayout::kSmem);
  if (e != cudaSuccess) return e;
  count_launch();
  kern<<<(unsigned)d.grid, kThreads, DLayout::kSmem, s>>>(tkm, tvm, tkl, tvl, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  count_launch();
  decode_combine_kernel<<<(unsigned)(a.B * a.Hkv), 32 * d.R, 0, s>>>(p, reinterpret_cast<__nv_bfloat16*>(a.O), a.lse);
  return cudaGetLastError();
}

}  // namespace msa
