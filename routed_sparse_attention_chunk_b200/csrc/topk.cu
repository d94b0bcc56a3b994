// Step 3 of the MSA memory path: the top-k documents of every query
// ("MSA: Memory Sparse Attention" README, "Architecture": select Top-k documents).
//
// Each document's score arrives as a 32-bit order-preserving key (see
// float_to_key).  Selection works on 64-bit keys
//     key = (score_key << 32) | (0xffffffff - doc)
// so that one unsigned comparison orders by score descending and, for equal
// scores, by lower document index first; padding is key 0, below every real key.
//
// Two passes of the same block routine: pass 1 splits each row into slices and
// keeps each slice's top-k; pass 2 merges the slices' candidates.  The block
// routine streams its input through shared memory in blocks of kSortN keys,
// keeping the running top-k at the front, and sorts each block with a bitonic
// network.  The top-k of a union is contained in the union of the parts'
// top-k, so the result is exact.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int kSortN = 2048;
constexpr int kSortThreads = 1024;

__device__ __forceinline__ void bitonic_desc(uint64_t* s) {
  for (int size = 2; size <= kSortN; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < kSortN / 2; i += blockDim.x) {
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

// FROM_DOC: the input is the [B, D] document key array (pass 1); otherwise the
// [B, nin] candidate keys of pass 1 (pass 2).
template <bool FROM_DOC>
__global__ void __launch_bounds__(kSortThreads)
topk_kernel(const uint32_t* __restrict__ doc_key, const uint64_t* __restrict__ cand_in,
            int64_t nin, int k, int nslice, uint64_t* __restrict__ cand_out,
            int32_t* __restrict__ out_idx, float* __restrict__ out_score) {
  __shared__ uint64_t s[kSortN];
  const int64_t b = blockIdx.y;
  const int slice = blockIdx.x;
  const int64_t per = (nin + nslice - 1) / nslice;
  const int64_t lo = (int64_t)slice * per;
  const int64_t hi = min(nin, lo + per);

  for (int i = threadIdx.x; i < k; i += blockDim.x) s[i] = 0ull;
  const int fresh = kSortN - k;
  for (int64_t base = lo; base < hi || base == lo; base += fresh) {
    __syncthreads();
    for (int i = threadIdx.x; i < fresh; i += blockDim.x) {
      const int64_t x = base + i;
      uint64_t key = 0ull;
      if (x < hi) {
        if (FROM_DOC)
          key = ((uint64_t)__ldg(doc_key + b * nin + x) << 32) | (uint64_t)(0xffffffffu - (uint32_t)x);
        else
          key = __ldg(cand_in + b * nin + x);
      }
      s[k + i] = key;
    }
    __syncthreads();
    bitonic_desc(s);
    if (base >= hi) break;
  }
  __syncthreads();
  if (cand_out) {
    for (int i = threadIdx.x; i < k; i += blockDim.x)
      cand_out[(b * nslice + slice) * k + i] = s[i];
  } else {
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
      const uint64_t key = s[i];
      out_idx[b * k + i] = (int32_t)(0xffffffffu - (uint32_t)(key & 0xffffffffu));
      if (out_score) out_score[b * k + i] = key_to_float((uint32_t)(key >> 32));
    }
  }
}

__global__ void decode_scores_kernel(const uint32_t* __restrict__ key, int64_t n, float* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = key_to_float(key[i]);
}

}  // namespace

int topk_num_slices(int64_t D, int k) {
  const int64_t fresh = kSortN - k;
  int64_t n = (D + fresh - 1) / fresh;
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
  if (a.nslice == 1) {
    count_launch();
    topk_kernel<true><<<dim3(1, (unsigned)a.B), kSortThreads, 0, s>>>(
        a.doc_key, nullptr, a.D, a.k, 1, nullptr, a.topk_idx, a.topk_score);
    return cudaGetLastError();
  }
  count_launch();
  topk_kernel<true><<<dim3(a.nslice, (unsigned)a.B), kSortThreads, 0, s>>>(
      a.doc_key, nullptr, a.D, a.k, a.nslice, a.cand, nullptr, nullptr);
  count_launch();
  topk_kernel<false><<<dim3(1, (unsigned)a.B), kSortThreads, 0, s>>>(
      nullptr, a.cand, (int64_t)a.nslice * a.k, a.k, 1, nullptr, a.topk_idx, a.topk_score);
  return cudaGetLastError();
}

}  // namespace msa
