// Launchers behind the C ABI (host side, C++ linkage).  Each returns the
// cudaError_t of its launches; the entry points in api.cu validate first.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "msa.h"

namespace msa {

// Counts every kernel launch of the library (read by msa_kernel_launch_count).
void count_launch(int n = 1);

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel on the stream is still running (once that kernel
// triggers its dependents, or exits), and must execute griddepcontrol.wait
// before it touches anything the previous kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

struct PoolArgs {
  const void *K, *V, *Kr;
  const int64_t *doc_tok_off, *doc_chunk_off;
  int64_t D, Ntok, C;
  int Hkv, d, Hr, dr, P;
  const float* rope_cs;
  int max_len;
  void *Kbar, *Vbar, *Krbar;
  float* kr_rnorm;
  int32_t* err_flag;
};
cudaError_t launch_pool(msa_dtype dt, const PoolArgs& a, cudaStream_t s);
cudaError_t launch_bank_rnorm(msa_dtype dt, const void* Krbar, int64_t C, int Hr, int dr,
                              float* kr_rnorm, cudaStream_t s);

struct RouteArgs {
  const void* Qr;
  int64_t B;
  int Tq, Hr, dr;
  const void* Krbar;
  const float* kr_rnorm;
  const int64_t* doc_chunk_off;
  int64_t D, C;
  uint32_t* doc_key;  // [B, D] ordered keys followed by [B] top-k counters, zeroed by the launcher
  float* rq;          // workspace [B * Tq, Hr]: 1 / ||Qr|| per row and head
  int32_t* chunk_doc; // workspace [C]: owning document of every chunk
  int32_t* err_flag;
};
cudaError_t launch_route(msa_dtype dt, const RouteArgs& a, cudaStream_t s);
// The argument checks msa_route_topk runs before it looks at its workspace (no launch, no
// pointer dereferenced): MSA_OK or the error msa_route_topk would return for these arguments.
msa_status route_topk_args_status(msa_dtype dt, const void* Qr, int64_t B, int Tq, int Hr, int dr,
                                  const void* Krbar, const float* kr_rnorm, const int64_t* doc_chunk_off,
                                  int64_t D, int64_t C, int k, const int32_t* topk_idx);

// Sum of each query's selected documents' recurrent states (the DGA layers'
// injected initial state): out[b] = sum_r states[idx[b, r]] in fp32.
cudaError_t launch_state_sum(msa_dtype dt, const void* states, int64_t D, int64_t S, const int32_t* idx,
                             int64_t B, int k, float* out, int32_t* err_flag, cudaStream_t s);

// Backward of the sparse attention (gradients in fp32; Drow is a workspace of
// [B, Hq, Tq] fp32 row dot products of dO and O).
struct AttnBwdArgs {
  const void *Q, *Kloc, *Vloc;
  int64_t B;
  int Tq, Lloc, Hq, Hkv, d;
  const void *Kmem, *Vmem;
  const int32_t* mem_len;
  int Mmax;
  float scale;
  const void *O, *dO;
  const float* lse;
  float *dQ, *dKloc, *dVloc, *dKmem, *dVmem;
  float* Drow;
  int32_t* err_flag;
};
size_t attn_bwd_workspace_size(int64_t B, int Tq, int Hq);
// Work split of the tensor-core dK / dV kernel (attn_bwd_tc.cu).  When a key
// tile's query steps span several chunks (max_chunks > 1) the kernel adds its
// partial dK / dV with atomics, so the outputs must be zeroed before it runs.
struct DkvPlan {
  bool applies;
  int chunk, max_chunks;
};
DkvPlan attn_dkv_tc_plan(msa_dtype dt, const AttnBwdArgs& a);
cudaError_t launch_attn_dkv_tc(msa_dtype dt, const AttnBwdArgs& a, const DkvPlan& pl, cudaStream_t s);
cudaError_t launch_attn_bwd(msa_dtype dt, const AttnBwdArgs& a, cudaStream_t s);

// Adjoint of the gather: dKbar / dVbar [C, Hkv, d] fp32 += the gathered rows' gradients.
struct GatherBwdArgs {
  const int32_t* topk_idx;
  int64_t B;
  int k;
  const int64_t* doc_chunk_off;
  int64_t D, C;
  const float *dKmem, *dVmem;
  const int32_t* mem_len;
  int Hkv, d, Mmax;
  float *dKbar, *dVbar;
  int32_t* err_flag;
};
cudaError_t launch_gather_bwd(const GatherBwdArgs& a, cudaStream_t s);

// Backward of the routing score of the selected documents (route_bwd.cu).
struct RouteBwdArgs {
  const void* Qr;
  int64_t B;
  int Tq, Hr, dr;
  const void* Krbar;
  const float* kr_rnorm;
  const int64_t* doc_chunk_off;
  int64_t D, C;
  int k;
  const int32_t* topk_idx;
  const float* d_score;
  float *dQr, *dKrbar;
  void* ws;  // route_bwd_workspace_size bytes
  int32_t* err_flag;
};
size_t route_bwd_workspace_size(int64_t B, int Tq, int k);
cudaError_t launch_route_bwd(msa_dtype dt, const RouteBwdArgs& a, cudaStream_t s);

// Top-k over ordered document keys [B, D]: writes idx / score (score may be null)
// and optionally decodes every document score into doc_scores.
struct TopkArgs {
  const uint32_t* doc_key;
  int64_t B, D;
  int k;
  uint64_t* cand;      // workspace [B, nslice, k]
  uint32_t* counters;  // workspace [B], zero on entry (the routing launcher clears it); left zero
  int nslice;
  int32_t* topk_idx;
  float* topk_score;
  float* doc_scores;
  int out_ld;  // row stride of topk_idx / topk_score (0: k)
};
int topk_num_slices(int64_t D, int k);
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s);
// Documents excl[b, 0..n) (row stride ld) of each query get key 0 (score -inf), so the
// top-k that follows passes them over while other documents remain; out-of-range
// entries are ignored.
cudaError_t launch_exclude(uint32_t* doc_key, int64_t B, int64_t D, const int32_t* excl, int ld, int n,
                           cudaStream_t s);

// Gated delta rule of the linear (DGA) layers' query path (gdr.cu), chunks of 64 tokens,
// one CTA per (value head, query); d = dk = dv = 128.
cudaError_t launch_gdr(msa_dtype dt, const void* q, const void* k, const void* v, const float* g, const float* beta,
                       int64_t B, int T, int Hk, int Hv, int d, const float* h0, float scale, void* o, float* hT,
                       cudaStream_t s);

// Round-to-round map of the memory interleave: out[r, :] = in[r, :] x W for rows
// r < rows (in [rows, K], W [K, N], out [rows, N]; fp32 accumulation, the
// result rounded to the storage type).
cudaError_t launch_project(msa_dtype dt, const void* in, const void* W, void* out, int64_t rows, int K, int N,
                           cudaStream_t s);

struct GatherArgs {
  const int32_t* topk_idx;
  int64_t B;
  int k;
  const int64_t* doc_chunk_off;
  int64_t D, C;
  const void *Kbar, *Vbar;
  int Hkv, d, Mmax;
  void *Kmem, *Vmem;
  int32_t* mem_len;
  int32_t* err_flag;
  bool host_src;  // Kbar / Vbar in page-locked host memory: few CTAs, many loads in flight each
  int idx_ld;     // row stride of topk_idx (0: k)
};
cudaError_t launch_gather(msa_dtype dt, const GatherArgs& a, cudaStream_t s);

// Segment plan of the index-driven attention (gather fused into attention):
// query b's selected chunks, in rank order, cut into segments of at most
// kSegRows consecutive chunk rows of one document.  Segment s of query b starts
// at bank row seg_row[b, s] and holds seg_cnt[b, s] valid rows; segments
// [nseg[b], Smax) are padding (row C, past the bank; count 0).  mem_len[b] is
// the number of selected rows kept (at most Mmax; more raises MSA_FLAG_OVERFLOW).
constexpr int kSegRows = 8;
struct PlanArgs {
  const int32_t* topk_idx;
  int64_t B;
  int k;
  const int64_t* doc_chunk_off;
  int64_t D, C;
  int Mmax, Smax;  // Smax: a multiple of 16, at least ceil(Mmax / 8) + k
  int32_t* seg_row;  // [B, Smax]
  uint8_t* seg_cnt;  // [B, Smax]
  int32_t* nseg;     // [B]
  int32_t* mem_len;  // [B]
  int32_t* err_flag;
  int idx_ld;        // row stride of topk_idx (0: k)
};
inline int plan_smax(int Mmax, int k) {
  const int s = (Mmax + kSegRows - 1) / kSegRows + k;
  return (s + 15) / 16 * 16;
}
cudaError_t launch_plan(const PlanArgs& a, cudaStream_t s);

// Memory rows are either dense [B, Mmax, Hkv, d] tensors (Kmem/Vmem), rows
// [0, mem_len[b]) used, or (seg_row != null) read in place from the bank
// K̄ / V̄ [C, Hkv, d] through a segment plan (Kmem/Vmem then point at the bank).
struct AttnArgs {
  const void *Q, *Kloc, *Vloc;
  int64_t B;
  int Tq, Lloc, Hq, Hkv, d;
  const void *Kmem, *Vmem;
  const int32_t* mem_len;   // [B]
  int Mmax;
  float scale;
  void* O;
  float* lse;
  void* ws;
  size_t ws_bytes;
  int32_t* err_flag;
  // index-driven memory rows (all null / 0 for dense Kmem / Vmem)
  const int32_t* seg_row;
  const uint8_t* seg_cnt;
  const int32_t* nseg;
  int Smax;
  int64_t C;  // bank rows
};
size_t attn_workspace_size(msa_dtype dt, int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, int Mmax);
cudaError_t launch_attn(msa_dtype dt, const AttnArgs& a, cudaStream_t s);
// Test hook of the prefill attention kernel's bounded waits (msa_testing_set_wait_polls).
void attn_tc_set_test_polls(int64_t polls);
// Whether a tensor-core kernel reads memory rows through a segment plan for this shape
// (bf16, d = 128, a decode or prefill shape those kernels take).
bool attn_indexed_applies(msa_dtype dt, const AttnArgs& a);
// Workspace of the decode kernel when the memory rows come through a plan of Smax segments.
size_t attn_indexed_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int Smax);

}  // namespace msa
