// Step 3 of the MSA memory path: the top-k documents of every query
// ("MSA: Memory Sparse Attention" README, "Architecture": select Top-k documents).
//
// Each document's score arrives as a 32-bit order-preserving key (see
// float_to_key).  Selection works on 64-bit keys
//     key = (score_key << 32) | (0xffffffff - doc)
// so that one unsigned comparison orders by score descending and, for equal
// scores, by lower document index first; padding is key 0, below every real key.
//
// One launch, grid (slices, B), 256 threads.  A slice of up to 8192 documents
// is held in registers, 32 keys per thread.  The threshold tau is the k-th
// largest of the 256 per-thread maxima: the k largest keys of the slice are all
// >= tau (k distinct thread maxima already are), and only the k threads whose
// maximum passes hold keys >= tau, so at most 32 k keys survive.  For k <= 32:
// each warp sorts its 32 maxima across lanes with shuffles and the eight sorted
// lists merge pairwise in three rounds (bitonic top-32 merges, half the warps
// per round) to give tau; larger k sorts the 256 maxima in shared memory.  The
// survivors are placed by a block-wide prefix sum of the threads' counts (one
// scan instead of a ballot and a shared atomic per key position); up to 32 are
// sorted in one warp's registers, more by a shared-memory bitonic sort, and
// more than 2048 (which needs k > 64) fall back to a block sort streamed over
// the slice.  With several slices, each slice's top-k goes to the workspace and
// the last CTA of the row to finish (an atomic counter, no waiting) merges the
// sorted lists.  (1024 threads and slices of 32768, one CTA per query of a 16M-
// token bank with no merge, ran slower: 64 busy SMs and register spills.)
// The top-k of a union is contained in the union of the parts' top-k, so the
// result is exact.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int kSortN = 2048;
constexpr int kSortThreads = 256;
constexpr int kPer = 32;                         // keys per thread in the filter
constexpr int kSlice = kSortThreads * kPer;      // documents per slice

__device__ __forceinline__ int next_pow2(int x) {
  int n = 1;
  while (n < x) n <<= 1;
  return n;
}

// Sort s[0, n) descending (n a power of two <= kSortN).
__device__ void bitonic_desc(uint64_t* s, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
        const int pos = 2 * i - (i & (stride - 1));
        const int par = pos + stride;
        const bool desc = (pos & size) == 0;
        const uint64_t x = s[pos], y = s[par];
        if ((x < y) == desc) {
          s[pos] = y;
          s[par] = x;
        }
      }
      __syncthreads();
    }
  }
}

// Top-k of n keys produced by load(i), i < n, left sorted in s[0, k).
template <typename Load>
__device__ void block_topk(uint64_t* s, int64_t n, int k, Load load) {
  for (int i = threadIdx.x; i < k; i += blockDim.x) s[i] = 0ull;
  const int fresh_max = kSortN - k;
  for (int64_t base = 0; base < n || base == 0; base += fresh_max) {
    const int fresh = (int)min((int64_t)fresh_max, max((int64_t)0, n - base));
    const int m = next_pow2(max(k + fresh, 2));
    __syncthreads();
    for (int i = threadIdx.x; i < m - k; i += blockDim.x) s[k + i] = i < fresh ? load(base + i) : 0ull;
    __syncthreads();
    bitonic_desc(s, m);
    if (base + fresh >= n) break;
  }
  __syncthreads();
}

__device__ __forceinline__ uint64_t doc_key64(uint32_t score_key, int64_t doc) {
  return ((uint64_t)score_key << 32) | (uint64_t)(0xffffffffu - (uint32_t)doc);
}

// 32 keys, one per lane, sorted descending across the warp (a bitonic network
// over lanes: no shared memory, no block barrier).
__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t x, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, x, stride);
      const bool desc = (lane & size) == 0 || size == 32;
      x = (((lane & stride) == 0) == desc) ? max(x, o) : min(x, o);
    }
  }
  return x;
}

// The 32 largest of two descending lane-lists, descending: a[i] against
// b[31 - i] keeps the top 32 as a bitonic sequence, which five compare-exchange
// steps sort.
__device__ __forceinline__ uint64_t warp_merge_top(uint64_t a, uint64_t b, int lane) {
  uint64_t x = max(a, __shfl_sync(0xffffffffu, b, 31 - lane));
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
    const uint64_t o = __shfl_xor_sync(0xffffffffu, x, stride);
    x = (lane & stride) == 0 ? max(x, o) : min(x, o);
  }
  return x;
}

// Top-k of keys row[lo, lo + n), n <= kSlice, left sorted in s[0, k); false
// when more than kSortN keys pass the filter (s is then clobbered).  wsum holds
// kSortThreads / 32 ints.
__device__ bool slice_topk_filter(uint64_t* s, int* wsum, const uint32_t* row, int64_t lo, int64_t n, int k) {
  constexpr int kWarps = kSortThreads / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // n <= kSlice: 32-bit indices; a key keeps only the low 32 bits of its document
  const int nn = (int)n;
  const uint32_t lo32 = (uint32_t)lo;
  auto key_of = [&](uint32_t sk, int i) -> uint64_t {
    return ((uint64_t)sk << 32) | (uint64_t)(0xffffffffu - (lo32 + (uint32_t)i));
  };
  // all 32 keys of this thread in registers from one round of loads
  uint32_t v[kPer];
#pragma unroll
  for (int m = 0; m < kPer; ++m) {
    const int i = tid + m * kSortThreads;
    v[m] = i < nn ? __ldg(row + lo + i) : 0u;
  }
  uint64_t mx = 0ull;
#pragma unroll
  for (int m = 0; m < kPer; ++m) {
    const int i = tid + m * kSortThreads;
    if (i < nn) mx = max(mx, key_of(v[m], i));
  }
  // tau = the k-th largest of the thread maxima
  uint64_t tau;
  if (k <= 32) {
    // each warp sorts its maxima; the sorted lists merge pairwise, half the warps a round
    uint64_t x = warp_sort_desc(mx, lane);
    s[tid] = x;
    __syncthreads();
#pragma unroll
    for (int half = kWarps / 2; half >= 1; half >>= 1) {
      if (warp < half) x = warp_merge_top(x, s[(warp + half) * 32 + lane], lane);
      __syncthreads();
      if (warp < half) s[tid] = x;
      __syncthreads();
    }
    tau = s[k - 1];
  } else {
    s[tid] = mx;
    __syncthreads();
    bitonic_desc(s, kSortThreads);
    tau = s[k - 1];
  }
  // keep the keys >= tau (the k thread maxima and what else their threads hold):
  // each thread counts its own, a block-wide exclusive prefix of the counts
  // gives where it writes them
  int c = 0;
#pragma unroll
  for (int m = 0; m < kPer; ++m) {
    const int i = tid + m * kSortThreads;
    c += (i < nn && key_of(v[m], i) >= tau) ? 1 : 0;
  }
  int inc = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();  // every thread has read tau from s, so s may be overwritten below
  int before = 0, total = 0;
  {
    const int w = lane < kWarps ? wsum[lane] : 0;
    int winc = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, winc, o);
      if (lane >= o) winc += t;
    }
    before = __shfl_sync(0xffffffffu, winc - w, warp & 31);
    total = __shfl_sync(0xffffffffu, winc, 31);
  }
  int pos = before + inc - c;
#pragma unroll
  for (int m = 0; m < kPer; ++m) {
    const int i = tid + m * kSortThreads;
    const uint64_t key = key_of(v[m], i);
    if (i < nn && key >= tau) {
      if (pos < kSortN) s[pos] = key;
      ++pos;
    }
  }
  __syncthreads();
  if (total > kSortN) return false;
  if (total <= 32) {  // one warp sorts the survivors in registers
    if (warp == 0) {
      const uint64_t x = warp_sort_desc(lane < total ? s[lane] : 0ull, lane);
      s[lane] = x;
    }
    __syncthreads();
    return true;
  }
  const int m2 = next_pow2(max(total, max(k, 2)));
  for (int i = total + tid; i < m2; i += kSortThreads) s[i] = 0ull;
  __syncthreads();
  bitonic_desc(s, m2);
  return true;
}

__global__ void __launch_bounds__(kSortThreads)
topk_kernel(const uint32_t* __restrict__ doc_key, int64_t D, int k, int nslice, uint64_t* cand,
            uint32_t* counters, int32_t* __restrict__ out_idx, float* __restrict__ out_score, int out_ld) {
  __shared__ uint64_t s[kSortN];
  __shared__ int wsum[kSortThreads / 32];
  __shared__ int last;
  pdl_wait();  // the scan's keys (launched as a programmatic dependent of it)
  const int64_t b = blockIdx.y;
  const int slice = blockIdx.x;
  const int64_t per = (D + nslice - 1) / nslice;
  const int64_t lo = (int64_t)slice * per;
  const int64_t n = max((int64_t)0, min(D, lo + per) - lo);
  const uint32_t* row = doc_key + b * D;
  // (the branch is uniform over the CTA)
  if (n > kSlice || !slice_topk_filter(s, wsum, row, lo, n, k)) {
    __syncthreads();
    block_topk(s, n, k, [&](int64_t i) -> uint64_t { return doc_key64(__ldg(row + lo + i), lo + i); });
  }
  if (nslice > 1) {
    // publish this slice's candidates; the last CTA of the row merges them
    for (int i = threadIdx.x; i < k; i += blockDim.x) cand[(b * nslice + slice) * k + i] = s[i];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(counters + b, 1u) == (unsigned)(nslice - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    const uint64_t* c = cand + b * nslice * k;
    if (k <= 32) {
      // every slice's list is sorted: the lists merge pairwise in rounds (half of them a
      // round, one warp per pair), up to kSortN / 32 lists at a time in shared memory
      constexpr int kLists = kSortN / 32;
      const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
      int have = 0, held = 0;  // slices merged so far; 1 once s[0, 32) holds their top list
      while (have < nslice) {
        const int take = min(nslice - have, kLists - held);
        for (int i = threadIdx.x; i < take * 32; i += kSortThreads) {
          const int l = i >> 5, e = i & 31;
          s[(held + l) * 32 + e] = e < k ? __ldcg(c + (int64_t)(have + l) * k + e) : 0ull;
        }
        __syncthreads();
        for (int L = held + take; L > 1;) {
          const int half = (L + 1) >> 1;
          // pairs (w, w + half); with L odd the middle list waits a round.  A warp writes only
          // list w < half, which no other warp of the round reads.
          for (int w = warp; w < L - half; w += kSortThreads / 32)
            s[w * 32 + lane] = warp_merge_top(s[w * 32 + lane], s[(w + half) * 32 + lane], lane);
          __syncthreads();
          L = half;
        }
        have += take;
        held = 1;
      }
    } else {
      block_topk(s, (int64_t)nslice * k, k, [&](int64_t i) -> uint64_t { return __ldcg(c + i); });
    }
    if (threadIdx.x == 0) counters[b] = 0u;  // ready for the next call on this workspace
  }
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    const uint64_t key = s[i];
    out_idx[b * out_ld + i] = (int32_t)(0xffffffffu - (uint32_t)(key & 0xffffffffu));
    if (out_score) out_score[b * out_ld + i] = key_to_float((uint32_t)(key >> 32));
  }
}

__global__ void exclude_kernel(uint32_t* __restrict__ doc_key, int64_t D, const int32_t* __restrict__ excl, int ld,
                               int n) {
  const int64_t b = blockIdx.x;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int32_t j = __ldg(excl + b * ld + i);
    if (j >= 0 && (int64_t)j < D) doc_key[b * D + j] = 0u;
  }
}

__global__ void decode_scores_kernel(const uint32_t* __restrict__ key, int64_t n, float* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = key_to_float(key[i]);
}

}  // namespace

int topk_num_slices(int64_t D, int k) {
  // slices the filter takes whole; capped so the merge stays a few blocks
  (void)k;
  int64_t n = (D + kSlice - 1) / kSlice;
  if (n < 1) n = 1;
  if (n > 1024) n = 1024;
  return (int)n;
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  if (a.doc_scores) {
    const int64_t n = a.B * a.D;
    const int64_t blocks = (n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096;
    count_launch();
    decode_scores_kernel<<<(unsigned)(blocks > 0 ? blocks : 1), 256, 0, s>>>(a.doc_key, n, a.doc_scores);
  }
  count_launch();
  return launch_pdl(topk_kernel, dim3(a.nslice, (unsigned)a.B), dim3(kSortThreads), 0, s, a.doc_key, a.D, a.k,
                    a.nslice, a.cand, a.counters, a.topk_idx, a.topk_score, a.out_ld > 0 ? a.out_ld : a.k);
}

cudaError_t launch_exclude(uint32_t* doc_key, int64_t B, int64_t D, const int32_t* excl, int ld, int n,
                           cudaStream_t s) {
  if (B <= 0 || n <= 0) return cudaSuccess;
  count_launch();
  exclude_kernel<<<(unsigned)B, 128, 0, s>>>(doc_key, D, excl, ld, n);
  return cudaGetLastError();
}

}  // namespace msa
