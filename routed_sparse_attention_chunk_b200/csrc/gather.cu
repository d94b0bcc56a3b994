// Step 4 of the MSA memory path: context assembly.
//
// "MSA: Memory Sparse Attention" README, "Inference Pipeline" stage 2: after
// Top-k, load only the selected K̄ / V̄ and concatenate them with the local
// context.  Query b's memory rows are the chunks of documents topk_idx[b, 0..k)
// in rank order, each document's chunks in ascending order.
//
// Every index is checked before it is used: a document outside [0, D) or a
// chunk range outside [0, C) is skipped and raises MSA_FLAG_INDEX_OOB; rows that
// do not fit in Mmax are dropped and raise MSA_FLAG_OVERFLOW.  Nothing traps.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tma_host.h"

namespace msa {
namespace {

struct Sel {
  int64_t cs, n;  // first chunk and chunk count of the selected document (n = 0: skipped)
};

// Rank r of query b in a selection list whose rows are ld entries apart.
__device__ __forceinline__ Sel selected(const int32_t* __restrict__ idx, const int64_t* __restrict__ off,
                                        int64_t D, int64_t C, int64_t b, int ld, int r, bool* bad) {
  const int32_t j = __ldg(idx + b * ld + r);
  if (j < 0 || (int64_t)j >= D) {
    *bad = true;
    return {0, 0};
  }
  const int64_t cs = __ldg(off + j), ce = __ldg(off + j + 1);
  if (cs < 0 || ce > C || ce < cs) {
    *bad = true;
    return {0, 0};
  }
  return {cs, ce - cs};
}

// One item per selected document (b, r).  Device banks: grid B * k, one item
// per CTA, with 8 loads of 16 bytes in flight per thread when there are fewer
// than two CTAs per SM (a single query's k documents: the copy is latency-bound)
// and 2 otherwise.  Host banks: a few CTAs loop over the items with 8 loads in
// flight per thread; that keeps the host link busy (it needs about 100 KB in
// flight) while leaving the SMs to the routing and attention of neighbouring
// batches, which would otherwise wait behind CTAs that spend their time on
// host-link latency.
constexpr int kHostCtas = 16;

template <int kUnroll>  // 16-byte loads in flight per thread and tensor
__global__ void __launch_bounds__(256) gather_kernel(GatherArgs a, int row_vecs) {
  const int64_t items = a.B * a.k;
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
    const int64_t b = item / a.k;
    const int r = (int)(item - b * a.k);
    const int ld = a.idx_ld > 0 ? a.idx_ld : a.k;
    bool bad = false;
    int64_t start = 0;
    for (int q = 0; q < r; ++q) start += selected(a.topk_idx, a.doc_chunk_off, a.D, a.C, b, ld, q, &bad).n;
    bool mine_bad = false;
    const Sel me = selected(a.topk_idx, a.doc_chunk_off, a.D, a.C, b, ld, r, &mine_bad);
    if (threadIdx.x == 0) {
      if (mine_bad) raise_flag(a.err_flag, MSA_FLAG_INDEX_OOB);
      if (r == a.k - 1) {
        const int64_t total = start + me.n;
        if (total > a.Mmax) raise_flag(a.err_flag, MSA_FLAG_OVERFLOW);
        a.mem_len[b] = (int32_t)(total < a.Mmax ? total : a.Mmax);
      }
    }
    if (r == a.k - 1) {
      // rows past the selection are zeroed: the attention kernels mask them, but a
      // masked weight of 0 times a non-finite value would still be NaN
      const int64_t total = min(start + me.n, (int64_t)a.Mmax);
      uint4* Kz = reinterpret_cast<uint4*>(a.Kmem) + (b * a.Mmax + total) * row_vecs;
      uint4* Vz = reinterpret_cast<uint4*>(a.Vmem) + (b * a.Mmax + total) * row_vecs;
      const int64_t nz = ((int64_t)a.Mmax - total) * row_vecs;
      for (int64_t i = threadIdx.x; i < nz; i += blockDim.x) {
        Kz[i] = make_uint4(0u, 0u, 0u, 0u);
        Vz[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    const int64_t n = min(me.n, max((int64_t)0, (int64_t)a.Mmax - start));
    if (n <= 0) continue;
    const uint4* Ks = reinterpret_cast<const uint4*>(a.Kbar) + me.cs * row_vecs;
    const uint4* Vs = reinterpret_cast<const uint4*>(a.Vbar) + me.cs * row_vecs;
    uint4* Kd = reinterpret_cast<uint4*>(a.Kmem) + (b * a.Mmax + start) * row_vecs;
    uint4* Vd = reinterpret_cast<uint4*>(a.Vmem) + (b * a.Mmax + start) * row_vecs;
    const int64_t nv = n * row_vecs;
    for (int64_t i0 = threadIdx.x; i0 < nv; i0 += (int64_t)blockDim.x * kUnroll) {
      uint4 kb[kUnroll], vb[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = i0 + (int64_t)u * blockDim.x;
        if (i < nv) {
          kb[u] = __ldg(Ks + i);
          vb[u] = __ldg(Vs + i);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = i0 + (int64_t)u * blockDim.x;
        if (i < nv) {
          Kd[i] = kb[u];
          Vd[i] = vb[u];
        }
      }
    }
  }
}

// Segment plan for the index-driven attention: one warp per query walks its k
// selected documents 32 at a time (a lane per document), prefix-sums their
// chunk counts across the warp to find where each document's rows start (rows
// past Mmax are dropped), and writes the document's rows as segments of at
// most kSegRows consecutive bank rows.  Entries past the query's last segment
// are padding: row C (past the end of the bank, which a TMA load reads as
// zeros) and count 0.
__global__ void __launch_bounds__(128) plan_kernel(PlanArgs a) {
  // the prefill attention kernel that reads the plan is launched as a programmatic
  // dependent: let it start its set-up now (it waits for this grid before reading)
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b = (int64_t)blockIdx.x * 4 + warp;
  if (b >= a.B) return;
  int32_t* row = a.seg_row + b * a.Smax;
  uint8_t* cnt = a.seg_cnt + b * a.Smax;
  const int ld = a.idx_ld > 0 ? a.idx_ld : a.k;
  int64_t rows_before = 0;  // selected rows of the earlier ranks (not truncated)
  int segs_before = 0;
  bool any_bad = false;
  for (int r0 = 0; r0 < a.k; r0 += 32) {
    const int r = r0 + lane;
    bool bad = false;
    const Sel me = r < a.k ? selected(a.topk_idx, a.doc_chunk_off, a.D, a.C, b, ld, r, &bad) : Sel{0, 0};
    any_bad |= bad;
    // inclusive prefix sums over the lanes of the chunk counts
    int64_t incl = me.n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int64_t start = rows_before + incl - me.n;
    const int64_t kept = max((int64_t)0, min(me.n, (int64_t)a.Mmax - start));
    const int segs = (int)((kept + kSegRows - 1) / kSegRows);
    int sincl = segs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, sincl, o);
      if (lane >= o) sincl += v;
    }
    const int s0 = segs_before + sincl - segs;
    for (int q = 0; q < segs; ++q) {
      const int si = s0 + q;
      if (si < a.Smax) {  // always true for Smax >= ceil(Mmax / 8) + k
        row[si] = (int32_t)(me.cs + (int64_t)q * kSegRows);
        cnt[si] = (uint8_t)min((int64_t)kSegRows, kept - (int64_t)q * kSegRows);
      }
    }
    rows_before += __shfl_sync(0xffffffffu, incl, 31);
    segs_before += __shfl_sync(0xffffffffu, sincl, 31);
  }
  const int ns = min(segs_before, a.Smax);
  for (int si = ns + lane; si < a.Smax; si += 32) {
    row[si] = (int32_t)a.C;
    cnt[si] = 0;
  }
  any_bad = __any_sync(0xffffffffu, any_bad);
  if (lane == 0) {
    if (any_bad) raise_flag(a.err_flag, MSA_FLAG_INDEX_OOB);
    if (rows_before > a.Mmax) raise_flag(a.err_flag, MSA_FLAG_OVERFLOW);
    a.nseg[b] = ns;
    a.mem_len[b] = (int32_t)min(rows_before, (int64_t)a.Mmax);
  }
}

}  // namespace

cudaError_t launch_plan(const PlanArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  count_launch();
  plan_kernel<<<(unsigned)((a.B + 3) / 4), 128, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gather(msa_dtype dt, const GatherArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  const int esz = dt == MSA_F32 ? 4 : 2;
  const int row_vecs = a.Hkv * a.d * esz / 16;
  const int64_t items = a.B * a.k;
  const unsigned grid = (unsigned)(a.host_src ? std::min<int64_t>(items, kHostCtas) : items);
  count_launch();
  if (a.host_src || items < 2 * (int64_t)sm_count())
    gather_kernel<8><<<grid, 256, 0, s>>>(a, row_vecs);
  else
    gather_kernel<2><<<grid, 256, 0, s>>>(a, row_vecs);
  return cudaGetLastError();
}

}  // namespace msa
