// Step 2 of the MSA memory path on the 5th-generation tensor cores: the
// routing scan of a bf16 bank.
//
// "MSA: Memory Sparse Attention" README, "Architecture": relevance is the
// cosine similarity of Q_r with the chunk-pooled K̄_r, mean-pooled over router
// heads, then the token-wise max; a document scores the max over its chunks.
//
//   S[c, r] = sum_h rk[c, h] rq[r, h] <K̄r[c, h], Qr[r, h]>        r = (b, t)
//   doc_key[b, doc(c)] = max over t, c of S[c, (b, t)] / Hr
//
// Design.  One work item is a tile of 128 chunks (the MMA's M, one TMEM lane
// per chunk) against a block of N query rows (the MMA's N).  For every router
// head h the tile's K̄r[., h, :] and the block's Qr[., h, :] arrive by TMA
// (128-byte swizzle), one tcgen05.mma chain (K = dr) writes the fp32 dot
// products of that head into the next of the TMEM accumulators (all 512
// columns: 8 of N = 64 or 4 of N = 128, so the tensor core can run a whole
// item ahead of the epilogue), and the epilogue warps fold rk * rq * dot into
// a register running sum.  The per-head cosine weights are why the
// heads cannot share one accumulator: the products stay exact (bf16 x bf16 in
// fp32) and every scale is applied in fp32 afterwards.  After the last head the
// epilogue takes the max over the block's tokens in registers, a segmented max
// over the warp's chunks of one document, and one atomicMax per document
// segment on an order-preserving key.
//
// Warp roles (320 threads, one CTA per SM, persistent over work items):
//   warp 0 lane 0  TMA producer (smem ring of STAGES head-slices)
//   warp 1         TMEM allocator; lane 0 issues the MMAs
//   warps 2..9     epilogue: two warpgroups, each reading half of the N columns
//                  of every TMEM lane quarter with one wait per head
// (the CTA-pair variant below has its own roles, thread count and work order)
// Every mbarrier wait is bounded; on expiry the kernel raises MSA_FLAG_TIMEOUT,
// drains its own copies and MMAs, frees TMEM and returns.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace msa {
namespace {

using namespace sm100;

constexpr int kTileM = 128;
constexpr int kThreads = 320;  // producer warp, MMA warp, 2 epilogue warpgroups
constexpr uint32_t kWaitPolls = 1u << 24;

struct RouteTcParams {
  const float* kr_rnorm;
  const float* rq;  // [rows, Hr]
  const int32_t* chunk_doc;  // [C] owning document of every chunk
  uint32_t* doc_key;
  int32_t* err_flag;
  int64_t D, C;
  int rows, Tq, Hr;
  int n_tiles, n_rb;
  int64_t items;
};

template <int DR, int N>
struct Layout {
  static constexpr int kBoxes = DR / 64;                  // 64-element (128-byte) K boxes per head
  static constexpr int kA = kTileM * DR * 2;              // K̄r slice of one head
  static constexpr int kB = N * DR * 2;                   // Qr slice of one head
  static constexpr int kStage = kA + kB;
  static constexpr int kStages = (200 * 1024) / kStage > 6 ? 6 : (200 * 1024) / kStage;
  static constexpr int kRq = 8 * 8 * (N / 2) * 4;         // per epilogue warp: rq of its columns, Hr <= 8
  static constexpr int kTr = 8 * 32 * 17 * 4;              // per epilogue warp: 32 chunks x 16 columns (+1 pad)
  static constexpr int kAcc = 512 / N;                      // fp32 accumulators of N columns in TMEM
  static constexpr int kBar = 8 * (2 * kStages + 2 * kAcc + 1) + 16;
  static constexpr int kSmem = 1024 + kStages * kStage + kRq + kTr + kBar;
  static_assert(kSmem <= 232448, "shared memory of one CTA");
  static constexpr uint32_t kTmemCols = 512;              // all of TMEM: kAcc accumulators
};

// Segmented max over the warp's lanes (consecutive chunks) grouped by document,
// then one atomicMax per document segment.
__device__ __forceinline__ void doc_max_atomic(float v, int doc, int lane, uint32_t* keys) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float vo = __shfl_down_sync(0xffffffffu, v, o);
    const int jo = __shfl_down_sync(0xffffffffu, doc, o);
    if (lane + o < 32 && jo == doc) v = fmaxf(v, vo);
  }
  const int jp = __shfl_up_sync(0xffffffffu, doc, 1);
  if (doc >= 0 && (lane == 0 || jp != doc)) atomicMax(keys + doc, float_to_key(v));
}

template <int DR, int N>
__global__ void __launch_bounds__(kThreads, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                RouteTcParams p) {
  using L = Layout<DR, N>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  float* rq_s = reinterpret_cast<float*>(smem + S * L::kStage);
  float* tr_s = reinterpret_cast<float*>(smem + S * L::kStage + L::kRq);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * L::kStage + L::kRq + L::kTr);
  uint64_t* full = bars;              // [S]   TMA -> MMA
  uint64_t* empty = bars + S;         // [S]   MMA -> TMA
  constexpr int NA = L::kAcc;
  uint64_t* accf = bars + 2 * S;      // [NA]  MMA -> epilogue
  uint64_t* acce = accf + NA;         // [NA]  epilogue -> MMA
  uint64_t* drain = acce + NA;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hr = p.Hr;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NA; ++i) {
      mbar_init(&accf[i], 1);
      mbar_init(&acce[i], 256);
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
  bool timed_out = false;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmQ);
      uint32_t it = 0;  // stage-fill counter
      for (int64_t item = blockIdx.x; item < p.items && !timed_out; item += gridDim.x) {
        const int tile = (int)(item / p.n_rb), rb = (int)(item % p.n_rb);
        for (int h = 0; h < Hr; ++h, ++it) {
          const uint32_t s = it % S, round = it / S;
          if (!mbar_wait(&empty[s], (round & 1) ^ 1, kWaitPolls)) {
            timed_out = true;
            break;
          }
          uint8_t* A = stage_base + s * L::kStage;
          uint8_t* Bq = A + L::kA;
          mbar_arrive_expect_tx(&full[s], L::kStage);
#pragma unroll
          for (int j = 0; j < L::kBoxes; ++j) {
            tma_load_2d(A + j * kTileM * 128, &tmK, h * DR + j * 64, tile * kTileM, &full[s]);
            tma_load_2d(Bq + j * N * 128, &tmQ, h * DR + j * 64, rb * N, &full[s]);
          }
        }
      }
      // drain: every stage's last fill must have landed before the CTA leaves
      const uint32_t fills = it;
      for (uint32_t s = 0; s < (uint32_t)S && s < fills; ++s) {
        const uint32_t last = (fills - 1 - s) / S * S + s;  // last fill index of stage s
        if (!mbar_wait(&full[s], (last / S) & 1, kWaitPolls)) timed_out = true;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTileM, N);
      uint32_t it = 0;
      for (int64_t item = blockIdx.x; item < p.items && !timed_out; item += gridDim.x) {
        for (int h = 0; h < Hr; ++h, ++it) {
          const uint32_t s = it % S, round = it / S;
          const uint32_t buf = it % NA, use = it / NA;
          if (!mbar_wait(&full[s], round & 1, kWaitPolls) || !mbar_wait(&acce[buf], (use & 1) ^ 1, kWaitPolls)) {
            timed_out = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(stage_base + s * L::kStage);
          const uint32_t b0 = a0 + L::kA;
          const uint32_t d = tmem + buf * N;
#pragma unroll
          for (int k = 0; k < DR / 16; ++k) {
            const int box = k >> 2, kk = k & 3;  // 4 K-steps of 16 per 128-byte row
            const uint64_t ad = desc_k_sw128(a0 + box * kTileM * 128 + kk * 32);
            const uint64_t bd = desc_k_sw128(b0 + box * N * 128 + kk * 32);
            mma_bf16_ss(d, ad, bd, idesc, k > 0 ? 1u : 0u);
          }
          mma_commit(&empty[s]);
          mma_commit(&accf[buf]);
        }
      }
      mma_commit(drain);
      if (!mbar_wait(drain, 0, kWaitPolls)) timed_out = true;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // two warpgroups; each covers all 128 TMEM lanes and half of the N columns
    constexpr int NH = N / 2;
    const int q = warp & 3;                 // TMEM lanes [32q, 32q + 32) belong to this warp
    const int wg = (warp - 2) >> 2;         // column half of this warpgroup
    const int col0 = wg * NH;
    float* rq_w = rq_s + (warp - 2) * 8 * NH;  // this warp's private copy (no cross-warp barrier)
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16) + col0;
    const float invHr = 1.0f / (float)Hr;
    // This lane's chunk of the next item: its document and its 1/||K̄r|| per
    // head are loaded one item ahead, so their latency overlaps the current
    // item's document walk instead of stalling the accumulator hand-off.
    int doc_n = -1;
    float rkv_n[8];
    auto prefetch = [&](int64_t item) {
      const int64_t cn = (item / p.n_rb) * kTileM + q * 32 + lane;
      const bool vn = item < p.items && cn < p.C;
      doc_n = vn ? __ldg(p.chunk_doc + cn) : -1;
#pragma unroll
      for (int h = 0; h < 8; ++h) rkv_n[h] = (vn && h < Hr) ? __ldg(p.kr_rnorm + cn * Hr + h) : 0.f;
    };
    // the routing prelude (keys zeroed, chunk map, query norms) must be done
    pdl_wait();
    prefetch(blockIdx.x);
    int rb_loaded = -1;  // query rows whose norms rq_w holds
    uint32_t it = 0;
    for (int64_t item = blockIdx.x; item < p.items && !timed_out; item += gridDim.x) {
      const int rb = (int)(item % p.n_rb);
      const int r0 = rb * N + col0;                 // first query row of this warp's columns
      const int nvalid = max(0, min(NH, p.rows - r0));
      if (rb != rb_loaded) {  // every item when the rows span several blocks, once otherwise
        __syncwarp();
        for (int i = lane; i < Hr * NH; i += 32) {
          const int h = i / NH, col = i - h * NH, r = r0 + col;
          rq_w[i] = r < p.rows ? __ldg(p.rq + (int64_t)r * Hr + h) : 0.f;
        }
        __syncwarp();
        rb_loaded = rb;
      }
      const int doc = doc_n;
      float rkv[8];  // this chunk's 1/||K̄r|| for every head
#pragma unroll
      for (int h = 0; h < 8; ++h) rkv[h] = rkv_n[h];
      float S_[NH];
#pragma unroll
      for (int j = 0; j < NH; ++j) S_[j] = 0.f;
      for (int h = 0; h < Hr; ++h, ++it) {
        const uint32_t buf = it % NA, use = it / NA;
        float rk = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) rk = i == h ? rkv[i] : rk;
        // the whole warp leaves together, so tcgen05.ld and the shuffles are never split
        if (!__all_sync(0xffffffffu, mbar_wait(&accf[buf], use & 1, kWaitPolls))) {
          timed_out = true;
          break;
        }
        tc_fence_after();
        float v[NH];
#pragma unroll
        for (int j0 = 0; j0 < NH; j0 += 16) tmem_ld16(lane_addr + buf * N + j0, *reinterpret_cast<float(*)[16]>(&v[j0]));
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&acce[buf]);  // the accumulator is in registers: the MMA may reuse it
        const float* rqh = rq_w + h * NH;
#pragma unroll
        for (int j = 0; j < NH; ++j) S_[j] = fmaf(v[j], rk * rqh[j], S_[j]);
      }
      if (timed_out) break;
      prefetch(item + gridDim.x);
      if (nvalid == 0) continue;
      const int b_first = r0 / p.Tq, b_last = (r0 + nvalid - 1) / p.Tq;
      if (b_first == b_last) {
        float m = -INFINITY;
#pragma unroll
        for (int j = 0; j < NH; ++j)
          if (j < nvalid) m = fmaxf(m, S_[j]);
        doc_max_atomic(m * invHr, doc, lane, p.doc_key + (int64_t)b_first * p.D);
      } else {
        // The columns belong to several queries (e.g. one token per query in
        // decode).  Transpose 16 columns at a time through shared memory so
        // that lane (16 * half + j) owns column j for the chunks of its half of
        // the warp, then walk those chunks in order: the document boundaries are
        // the same for every lane, so the walk is warp-uniform and a document
        // segment ends in one atomicMax per column.  A document that straddles
        // the two halves gets two atomics, which max-combine.
        float* tr = tr_s + (warp - 2) * 32 * 17;
        const int hf = lane >> 4, jl = lane & 15;
#pragma unroll
        for (int h0 = 0; h0 < NH; h0 += 16) {
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 16; ++j) tr[lane * 17 + j] = S_[h0 + j];
          __syncwarp();
          const bool colv = h0 + jl < nvalid;
          const int b = colv ? (r0 + h0 + jl) / p.Tq : 0;
          uint32_t* keys = p.doc_key + (int64_t)b * p.D;
          int cur = __shfl_sync(0xffffffffu, doc, 16 * hf);
          float m = -INFINITY;
#pragma unroll
          for (int ii = 0; ii < 16; ++ii) {
            const int i = 16 * hf + ii;
            m = fmaxf(m, tr[i * 17 + jl]);
            const int nd = ii + 1 < 16 ? __shfl_sync(0xffffffffu, doc, i + 1) : -2;
            if (nd != cur) {
              if (colv && cur >= 0) atomicMax(keys + cur, float_to_key(m * invHr));
              m = -INFINITY;
              cur = nd;
            }
          }
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

template <int DR, int N>
cudaError_t launch_t(const RouteArgs& a, cudaStream_t s) {
  using L = Layout<DR, N>;
  const int rows = (int)(a.B * a.Tq);
  CUtensorMap tmK, tmQ;
  if (!make_tmap_2d_bf16(&tmK, a.Krbar, (uint64_t)a.Hr * DR, (uint64_t)a.C, (uint64_t)a.Hr * DR * 2, 64, kTileM) ||
      !make_tmap_2d_bf16(&tmQ, a.Qr, (uint64_t)a.Hr * DR, (uint64_t)rows, (uint64_t)a.Hr * DR * 2, 64, N))
    return cudaErrorInvalidValue;
  RouteTcParams p;
  p.kr_rnorm = a.kr_rnorm;
  p.rq = a.rq;
  p.chunk_doc = a.chunk_doc;
  p.doc_key = a.doc_key;
  p.err_flag = a.err_flag;
  p.D = a.D;
  p.C = a.C;
  p.rows = rows;
  p.Tq = a.Tq;
  p.Hr = a.Hr;
  p.n_tiles = (int)((a.C + kTileM - 1) / kTileM);
  p.n_rb = (rows + N - 1) / N;
  p.items = (int64_t)p.n_tiles * p.n_rb;
  if (p.items == 0) return cudaGetLastError();
  cudaError_t e = cudaFuncSetAttribute(route_tc_kernel<DR, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  const int64_t grid = p.items < sm_count() ? p.items : sm_count();
  count_launch();
  return launch_pdl(route_tc_kernel<DR, N>, dim3((unsigned)grid), dim3(kThreads), (size_t)L::kSmem, s, tmK, tmQ, p);
}


// ------------------------------------------------------------------ CTA pairs
// Long queries (many rows of one query, e.g. a 4096-token prefill) make the
// scan a dense contraction.  On one CTA (M = N = 128) the tensor core reads
// 128 B of operands from shared memory per clock while the TMA writes the next
// operands into the same memory, and a clock64 timeline showed each head's MMAs
// taking ~1.8x their ideal time.  A cluster of two CTAs runs one MMA of M = 256
// chunks x N = 256 query rows per head instead: each CTA holds its own 128
// chunks of K̄r and 128 of the rows, the leader issues the MMA for both, and
// each CTA's tensor memory receives its 128 chunks x all 256 rows, which halves
// the shared-memory operand bytes per flop.  Per head the accumulator is 256
// TMEM columns, double-buffered; each of the two epilogue warpgroups of a CTA
// keeps 128 running sums per thread.  Used when every block of 256 rows
// belongs to one query (one query, or Tq a multiple of 256).
//
// Work order: each pair takes one contiguous range of items, enumerated in
// groups of kGroup tile pairs, row block by row block within a group; a pair
// so reloads its rows' norms only when the row block changes, and the group's
// K̄r (kGroup x 512 KB) stays in L2 while the row blocks pass over it.
//
// Handshakes: both CTAs' copies of a stage complete on the leader's `full`
// barrier (the leader arms it for both); the leader's commits arrive on the
// `empty` and `accf` barriers of both CTAs; both CTAs' epilogue warps arrive on
// the leader's `acce` barrier.  A cluster barrier after set-up and before
// teardown orders barrier initialisation, TMEM allocation and the last MMAs.
// Packed pairs of fp32 (sm_100 f32x2 arithmetic: one instruction for two values).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

template <int DR>
struct PairLayout {
  static constexpr int kRowsPerCta = 128;                 // query rows each CTA loads (N / 2)
  static constexpr int kN = 2 * kRowsPerCta;              // the MMA's N
  static constexpr int kBoxes = DR / 64;
  static constexpr int kA = kTileM * DR * 2;
  static constexpr int kB = kRowsPerCta * DR * 2;
  static constexpr int kStage = kA + kB;
  static constexpr int kStages = (192 * 1024) / kStage > 6 ? 6 : (192 * 1024) / kStage;
  static constexpr int kNH = kN / 2;                      // columns per epilogue warpgroup
  static_assert(kNH % 64 == 0, "the epilogue reads its columns 64 at a time and frees the accumulator after the last 64");
  static constexpr int kRq = 8 * 8 * kNH * 4;             // per epilogue warp: rq of its columns, Hr <= 8
  static constexpr int kBar = 8 * (2 * kStages + 2 * 2 + 1) + 16;
  static constexpr int kSmem = 1024 + kStages * kStage + kRq + kBar;
  static_assert(kSmem <= 232448, "shared memory of one CTA");
  static constexpr uint32_t kTmemCols = 512;              // two accumulators of kN columns
};
constexpr int kGroup = 8;  // tile pairs per work group

// 384 threads: warpgroup 0 (TMA producer, TMEM owner / MMA issuer, two idle
// warps) gives registers to the two epilogue warpgroups, whose 128 running sums
// per thread do not fit the 168 registers a thread gets at launch.
constexpr int kPairThreads = 384;
constexpr uint32_t kRegsControl = 40, kRegsEpilogue = 232;
constexpr uint32_t kPairRegsNeeded = 128 * kRegsControl + 256 * kRegsEpilogue;

// Item at position L of the work order: (tile pair, row block).  The host
// keeps the item count below 2^31, so 32-bit arithmetic suffices.
__device__ __forceinline__ void pair_item(uint32_t L, const RouteTcParams& p, int& tile, int& rb) {
  const uint32_t per_group = (uint32_t)kGroup * (uint32_t)p.n_rb;
  const uint32_t g = L / per_group;
  const uint32_t w = L - g * per_group;
  const uint32_t tg = (uint32_t)min(kGroup, p.n_tiles - (int)g * kGroup);
  rb = (int)(w / tg);
  tile = (int)(g * kGroup + (w - (uint32_t)rb * tg));
}

template <int DR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
route_tc_pair_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                     RouteTcParams p) {
  using L = PairLayout<DR>;
  constexpr int S = L::kStages;
  constexpr int NH = L::kNH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  float* rq_s = reinterpret_cast<float*>(smem + S * L::kStage);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * L::kStage + L::kRq);
  uint64_t* full = bars;          // [S]  leader: both CTAs' copies of a stage landed
  uint64_t* empty = bars + S;     // [S]  each CTA: the MMA is done with its stage
  uint64_t* accf = bars + 2 * S;  // [2]  each CTA: accumulator ready
  uint64_t* acce = accf + 2;      // [2]  leader: both CTAs' epilogues have read it
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int64_t per = (p.items + npairs - 1) / npairs;
  const int64_t L0 = pair * per, L1 = min(p.items, L0 + per);  // this pair's items
  const int Hr = p.Hr;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accf[i], 1);
      mbar_init(&acce[i], 2 * 8);  // one arrival per epilogue warp of either CTA
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();

  if (warp < 4) {
    setmaxnreg_dec<kRegsControl>();
    const uint32_t tmem = *tmem_slot;
    bool timed_out = false;
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- TMA producer (both CTAs)
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmQ);
      const uint32_t full0 = mapa_shared(smem_u32(full), 0);
      uint32_t it = 0;
      for (int64_t Li = L0; Li < L1 && !timed_out; ++Li) {
        int tile, rb;
        pair_item(Li, p, tile, rb);
        const int ychunk = tile * 2 * kTileM + (int)rank * kTileM;
        const int yrow = rb * L::kN + (int)rank * L::kRowsPerCta;
        for (int h = 0; h < Hr; ++h, ++it) {
          const uint32_t s = it % S, round = it / S;
          if (!mbar_wait(&empty[s], (round & 1) ^ 1, kWaitPolls)) {
            timed_out = true;
            break;
          }
          uint8_t* A = stage_base + s * L::kStage;
          uint8_t* Bq = A + L::kA;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * L::kStage);
#pragma unroll
          for (int j = 0; j < L::kBoxes; ++j) {
            tma_load_2d_pair(A + j * kTileM * 128, &tmK, h * DR + j * 64, ychunk, full0 + 8u * s);
            tma_load_2d_pair(Bq + j * L::kRowsPerCta * 128, &tmQ, h * DR + j * 64, yrow, full0 + 8u * s);
          }
        }
      }
      if (rank == 0) {
        // every stage's last fill (both CTAs' copies) must have landed before teardown
        const uint32_t fills = it;
        for (uint32_t s = 0; s < (uint32_t)S && s < fills; ++s) {
          const uint32_t last = (fills - 1 - s) / S * S + s;
          if (!mbar_wait(&full[s], (last / S) & 1, kWaitPolls)) timed_out = true;
        }
      } else if (timed_out) {
        // this CTA's copies complete on the leader's barriers; give any still in
        // flight time to land before the pair tears down
        for (int i = 0; i < 2000; ++i) __nanosleep(1000);
      }
    } else if (warp == 1 && lane == 0 && rank == 0) {
      // ---------------------------------------------------------- MMA issuer (leader)
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kTileM, L::kN);
      uint32_t it = 0;
      for (int64_t Li = L0; Li < L1 && !timed_out; ++Li) {
        for (int h = 0; h < Hr; ++h, ++it) {
          const uint32_t s = it % S, round = it / S;
          const uint32_t buf = it & 1, use = it >> 1;
          if (!mbar_wait(&full[s], round & 1, kWaitPolls) ||
              !mbar_wait(&acce[buf], (use & 1) ^ 1, kWaitPolls)) {
            timed_out = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(stage_base + s * L::kStage);
          const uint32_t b0 = a0 + L::kA;
          const uint32_t d = tmem + buf * L::kN;
#pragma unroll
          for (int k = 0; k < DR / 16; ++k) {
            const int box = k >> 2, kk = k & 3;
            const uint64_t ad = desc_k_sw128(a0 + box * kTileM * 128 + kk * 32);
            const uint64_t bd = desc_k_sw128(b0 + box * L::kRowsPerCta * 128 + kk * 32);
            mma_bf16_ss_pair(d, ad, bd, idesc, k > 0 ? 1u : 0u);
          }
          mma_commit_pair(&empty[s], 3);
          mma_commit_pair(&accf[buf], 3);
        }
      }
      mma_commit_pair(drain, 1);
      if (!mbar_wait(drain, 0, kWaitPolls)) timed_out = true;
    }
    if (timed_out) raise_flag(p.err_flag, MSA_FLAG_TIMEOUT);
  } else {
    setmaxnreg_inc<kRegsEpilogue>();
    // ------------------------------------------------------------ epilogue (both CTAs)
    const uint32_t tmem = *tmem_slot;
    bool timed_out = false;
    const int q = warp & 3;
    const int wg = (warp - 4) >> 2;
    const int col0 = wg * NH;
    float* rq_w = rq_s + (warp - 4) * 8 * NH;
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16) + col0;
    const uint32_t acce0 = mapa_shared(smem_u32(acce), 0);
    const float invHr = 1.0f / (float)Hr;
    pdl_wait();  // the routing prelude (keys, chunk map, query norms) is done
    int rb_loaded = -1;
    uint32_t it = 0;
    for (int64_t Li = L0; Li < L1 && !timed_out; ++Li) {
      int tile, rb;
      pair_item(Li, p, tile, rb);
      const int r0 = rb * L::kN + col0;  // column j of this warpgroup is query row r0 + j
      const int nvalid = max(0, min(NH, p.rows - r0));
      if (rb != rb_loaded) {
        // the rows' 1/||Qr|| per head: every load issued before any is stored
        float t[NH / 32][8];
#pragma unroll
        for (int k = 0; k < NH / 32; ++k) {
          const int r = r0 + k * 32 + lane;
#pragma unroll
          for (int h = 0; h < 8; ++h) t[k][h] = (r < p.rows && h < Hr) ? __ldg(p.rq + (int64_t)r * Hr + h) : 0.f;
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < NH / 32; ++k)
#pragma unroll
          for (int h = 0; h < 8; ++h) rq_w[h * NH + k * 32 + lane] = t[k][h];
        __syncwarp();
        rb_loaded = rb;
      }
      // this lane's chunk: its document and, per head, 1 / ||K̄r||
      const int64_t cn = (int64_t)tile * 2 * kTileM + rank * kTileM + q * 32 + lane;
      const bool cvalid = cn < p.C;
      const int doc = cvalid ? __ldg(p.chunk_doc + cn) : -1;
      const float* rkp = p.kr_rnorm + (cvalid ? cn : 0) * Hr;
      float S_[NH];
#pragma unroll
      for (int j = 0; j < NH; ++j) S_[j] = 0.f;
      for (int h = 0; h < Hr; ++h, ++it) {
        const uint32_t buf = it & 1, use = it >> 1;
        const float rk = cvalid ? __ldg(rkp + h) : 0.f;  // issued before the wait, used after it
        if (!__all_sync(0xffffffffu, mbar_wait(&accf[buf], use & 1, kWaitPolls))) {
          timed_out = true;
          break;
        }
        tc_fence_after();
        const float* rqh = rq_w + h * NH;
        const uint64_t rk2 = f2_pack(rk, rk);
        // 64 columns per tensor-memory wait (the load latency is paid twice per head)
#pragma unroll
        for (int j0 = 0; j0 < NH; j0 += 64) {
          float v[64];
#pragma unroll
          for (int c = 0; c < 64; c += 16)
            tmem_ld16(lane_addr + buf * L::kN + j0 + c, *reinterpret_cast<float(*)[16]>(&v[c]));
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 64; c += 16) tmem_regs_ready(*reinterpret_cast<float(*)[16]>(&v[c]));
          if (j0 + 64 == NH) {
            // the whole accumulator is in registers: the leader's MMA may reuse it
            // while this half's products are summed
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(acce0 + 8u * buf);
          }
#pragma unroll
          for (int j4 = 0; j4 < 64; j4 += 4) {
            const float4 w = *reinterpret_cast<const float4*>(rqh + j0 + j4);
            // rk * rq for four columns in two packed multiplies, then one fma per column
            float k0, k1, k2, k3;
            f2_unpack(f2_mul(f2_pack(w.x, w.y), rk2), k0, k1);
            f2_unpack(f2_mul(f2_pack(w.z, w.w), rk2), k2, k3);
            S_[j0 + j4] = fmaf(v[j4], k0, S_[j0 + j4]);
            S_[j0 + j4 + 1] = fmaf(v[j4 + 1], k1, S_[j0 + j4 + 1]);
            S_[j0 + j4 + 2] = fmaf(v[j4 + 2], k2, S_[j0 + j4 + 2]);
            S_[j0 + j4 + 3] = fmaf(v[j4 + 3], k3, S_[j0 + j4 + 3]);
          }
        }
      }
      if (timed_out) break;
      if (nvalid == 0) continue;
      float m = -INFINITY;
      if (nvalid == NH) {  // the usual case: a tree of maxima over all columns
#pragma unroll
        for (int w = NH / 2; w >= 1; w /= 2)
#pragma unroll
          for (int j = 0; j < w; ++j) S_[j] = fmaxf(S_[j], S_[j + w]);
        m = S_[0];
      } else {
#pragma unroll
        for (int j = 0; j < NH; ++j)
          if (j < nvalid) m = fmaxf(m, S_[j]);
      }
      doc_max_atomic(m * invHr, doc, lane, p.doc_key + (int64_t)(r0 / p.Tq) * p.D);
    }
    if (timed_out) raise_flag(p.err_flag, MSA_FLAG_TIMEOUT);
  }

  // teardown: nothing from the role branches is live here
  tc_fence_before();
  cluster_sync_all();
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc_pair(*reinterpret_cast<volatile uint32_t*>(tmem_slot), L::kTmemCols);
  }
}

template <int DR>
cudaError_t launch_pair_t(const RouteArgs& a, cudaStream_t s) {
  using L = PairLayout<DR>;
  const int rows = (int)(a.B * a.Tq);
  RouteTcParams p;
  p.kr_rnorm = a.kr_rnorm;
  p.rq = a.rq;
  p.chunk_doc = a.chunk_doc;
  p.doc_key = a.doc_key;
  p.err_flag = a.err_flag;
  p.D = a.D;
  p.C = a.C;
  p.rows = rows;
  p.Tq = a.Tq;
  p.Hr = a.Hr;
  p.n_tiles = (int)((a.C + 2 * kTileM - 1) / (2 * kTileM));  // pairs of 128-chunk tiles
  p.n_rb = (rows + L::kN - 1) / L::kN;
  p.items = (int64_t)p.n_tiles * p.n_rb;
  if (p.items == 0) return cudaGetLastError();
  if (p.items > 0x7fffffffLL) return launch_t<DR, 128>(a, s);  // the work order is 32-bit
  auto kern = route_tc_pair_kernel<DR>;
  // The register split may only hand out what the launch allocated; a build
  // that gives the kernel fewer registers per thread takes the one-CTA scan.
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if ((uint32_t)fa.numRegs * kPairThreads < kPairRegsNeeded) return launch_t<DR, 128>(a, s);
  CUtensorMap tmK, tmQ;
  if (!make_tmap_2d_bf16(&tmK, a.Krbar, (uint64_t)a.Hr * DR, (uint64_t)a.C, (uint64_t)a.Hr * DR * 2, 64, kTileM) ||
      !make_tmap_2d_bf16(&tmQ, a.Qr, (uint64_t)a.Hr * DR, (uint64_t)rows, (uint64_t)a.Hr * DR * 2, 64,
                         L::kRowsPerCta))
    return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  // as many pairs as can be resident at once (each CTA fills an SM)
  static int max_pairs[2] = {0, 0};
  int& mp = max_pairs[DR == 128 ? 1 : 0];
  if (mp == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * (sm_count() / 2)));
    cfg.blockDim = dim3(kPairThreads);
    cfg.dynamicSmemBytes = L::kSmem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      n = sm_count() / 2;
    }
    mp = n;
  }
  const int64_t pairs = p.items < mp ? p.items : mp;
  count_launch();
  return launch_pdl(kern, dim3((unsigned)(2 * pairs)), dim3(kPairThreads), (size_t)L::kSmem, s, tmK, tmQ, p);
}

}  // namespace

bool route_tc_applies(const RouteArgs& a) {
  if (a.Hr < 1 || a.Hr > 8 || (a.dr != 64 && a.dr != 128) || a.C < 1) return false;
  return a.C <= 0x7fffffffLL - kTileM && a.B * a.Tq <= 0x7fffffffLL;
}

// The caller has zeroed the keys, built chunk_doc and the query norms rq (the
// routing prelude); the TMA maps need 16-byte aligned bases (checked by the
// entry point).
cudaError_t launch_route_tc(const RouteArgs& a, cudaStream_t s) {
  const int64_t rows = a.B * a.Tq;
  // CTA pairs when every block of 256 rows lies inside one query
  if (rows >= 256 && (a.B == 1 || a.Tq % 256 == 0))
    return a.dr == 128 ? launch_pair_t<128>(a, s) : launch_pair_t<64>(a, s);
  if (a.dr == 128) return rows <= 64 ? launch_t<128, 64>(a, s) : launch_t<128, 128>(a, s);
  return rows <= 64 ? launch_t<64, 64>(a, s) : launch_t<64, 128>(a, s);
}

}  // namespace msa
