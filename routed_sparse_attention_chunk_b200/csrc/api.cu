// The C ABI of the MSA memory-path library: argument checks, workspace
// carving, and dispatch to the launchers.  Nothing here allocates or
// synchronises; every launch goes to the caller's stream.
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "internal.h"
#include "msa.h"

using namespace msa;

namespace msa {
static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace msa

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// True when kernels may dereference p as it is: device or managed memory, or
// page-locked host memory mapped at the same address (unified addressing).
// Pageable host memory (and anything the runtime does not know) is refused, so
// a misplaced host pointer is an argument error, not a device fault.
bool device_readable(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) return true;
  return at.type == cudaMemoryTypeHost && at.devicePointer == p;
}
// Page-locked host memory the device reads in place (the host tier of K̄ / V̄).
bool host_resident(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeHost;
}
inline bool head_dim_ok(int d) { return d == 64 || d == 128; }
inline bool dtype_ok(msa_dtype dt) { return dt == MSA_F32 || dt == MSA_BF16; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
constexpr int64_t kMaxIndex = 0x7fffffff;
constexpr int kMaxK = 256;

inline msa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

struct RouteWs {
  uint32_t* doc_key;
  uint64_t* cand;
  float* rq;
  int32_t* chunk_doc;
  int nslice;
  size_t bytes;
};

RouteWs route_ws_layout(void* base, int64_t B, int Tq, int Hr, int64_t D, int64_t C, int k) {
  RouteWs w{};
  w.nslice = topk_num_slices(D, k);
  const size_t keys = round_up(sizeof(uint32_t) * ((size_t)B * (size_t)D + (size_t)B), 256);  // + counters
  const size_t cand = w.nslice > 1 ? round_up(sizeof(uint64_t) * (size_t)B * w.nslice * k, 256) : 0;
  const size_t rq = round_up(sizeof(float) * (size_t)B * (size_t)Tq * (size_t)Hr, 256);
  const size_t cdoc = round_up(sizeof(int32_t) * (size_t)(C > 0 ? C : 1), 256);
  w.bytes = keys + cand + rq + cdoc;
  if (base) {
    w.doc_key = reinterpret_cast<uint32_t*>(base);
    w.cand = cand ? reinterpret_cast<uint64_t*>(static_cast<char*>(base) + keys) : nullptr;
    w.rq = reinterpret_cast<float*>(static_cast<char*>(base) + keys + cand);
    w.chunk_doc = reinterpret_cast<int32_t*>(static_cast<char*>(base) + keys + cand + rq);
  }
  return w;
}

msa_status check_route(msa_dtype dt, const void* Qr, int64_t B, int Tq, int Hr, int dr, const void* Krbar,
                       const float* kr_rnorm, const int64_t* doc_chunk_off, int64_t D, int64_t C, int k,
                       const int32_t* topk_idx) {
  if (!dtype_ok(dt)) return MSA_ERR_INVALID_ARG;
  if (B < 0 || Tq < 1 || D < 1 || C < 0 || D > kMaxIndex || C > kMaxIndex) return MSA_ERR_INVALID_ARG;
  if (k < 1 || k > D) return MSA_ERR_INVALID_ARG;
  if (k > kMaxK || !head_dim_ok(dr) || Hr < 1 || Hr > 8) return MSA_ERR_UNSUPPORTED;
  if (!Qr || !Krbar || !kr_rnorm || !doc_chunk_off || !topk_idx) return MSA_ERR_INVALID_ARG;
  if (!aligned16(Qr) || !aligned16(Krbar)) return MSA_ERR_INVALID_ARG;
  if (B * (int64_t)Tq > kMaxIndex) return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

msa_status check_attn(msa_dtype dt, const void* Q, const void* Kloc, const void* Vloc, int64_t B, int Tq,
                      int Lloc, int Hq, int Hkv, int d, int Mmax) {
  if (!dtype_ok(dt)) return MSA_ERR_INVALID_ARG;
  if (B < 0 || Tq < 1 || Lloc < Tq || Hkv < 1 || Hq < 1 || Hq % Hkv != 0 || Mmax < 0) return MSA_ERR_INVALID_ARG;
  if (!head_dim_ok(d)) return MSA_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return MSA_ERR_UNSUPPORTED;  // grid y / z limits
  if ((int64_t)Mmax + Lloc > kMaxIndex) return MSA_ERR_INVALID_ARG;
  if (!Q || !Kloc || !Vloc) return MSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(Kloc) || !aligned16(Vloc)) return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

// Workspace of msa_sparse_attn_indexed: the segment plan, then either the
// decode kernel's partial results (index-driven attention) or, for shapes and
// banks the tensor-core kernels do not read in place, the gathered rows (sized
// for fp32 storage) and the dense attention's workspace.
struct IndexedWs {
  int Smax;
  int32_t *seg_row, *nseg, *mem_len;
  uint8_t* seg_cnt;
  void *attn_ws, *Kmem, *Vmem, *dense_ws;
  size_t attn_ws_bytes, dense_ws_bytes, bytes;
};

IndexedWs indexed_ws_layout(void* base, int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, int k, int Mmax) {
  IndexedWs w{};
  w.Smax = plan_smax(Mmax, k);
  const size_t rows = round_up(sizeof(int32_t) * (size_t)B * w.Smax, 256);
  const size_t cnts = round_up((size_t)B * w.Smax, 256);
  const size_t per_b = round_up(sizeof(int32_t) * (size_t)B, 256);
  const size_t plan = rows + cnts + 2 * per_b;
  w.attn_ws_bytes = round_up(attn_indexed_workspace_size(B, Tq, Lloc, Hq, Hkv, w.Smax), 256);
  const size_t mem = round_up(sizeof(float) * (size_t)B * (size_t)Mmax * (size_t)Hkv * (size_t)d, 256);
  w.dense_ws_bytes = round_up(attn_workspace_size(MSA_BF16, B, Tq, Lloc, Hq, Hkv, d, Mmax), 256);
  const size_t dense = 2 * mem + w.dense_ws_bytes;
  w.bytes = plan + (w.attn_ws_bytes > dense ? w.attn_ws_bytes : dense);
  if (base) {
    char* p = static_cast<char*>(base);
    w.seg_row = reinterpret_cast<int32_t*>(p);
    w.seg_cnt = reinterpret_cast<uint8_t*>(p + rows);
    w.nseg = reinterpret_cast<int32_t*>(p + rows + cnts);
    w.mem_len = reinterpret_cast<int32_t*>(p + rows + cnts + per_b);
    w.attn_ws = p + plan;
    w.Kmem = p + plan;
    w.Vmem = p + plan + mem;
    w.dense_ws = p + plan + 2 * mem;
  }
  return w;
}

msa_status check_indexed(const int32_t* topk_idx, int k, const int64_t* doc_chunk_off, int64_t D, int64_t C,
                         const void* Kbar, const void* Vbar) {
  if (k < 1 || D < 1 || C < 0 || D > kMaxIndex || C > kMaxIndex) return MSA_ERR_INVALID_ARG;
  if (k > 65535) return MSA_ERR_UNSUPPORTED;
  if (!topk_idx || !doc_chunk_off || !Kbar || !Vbar) return MSA_ERR_INVALID_ARG;
  if (!aligned16(Kbar) || !aligned16(Vbar)) return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

// Steps 4 + 5 once the arguments are checked: the index-driven attention when the
// tensor-core kernels take the shape and the bank is in device memory, else the
// gather into the workspace followed by the dense attention.
msa_status run_indexed(msa_dtype dt, const void* Q, const void* Kloc, const void* Vloc, int64_t B, int Tq, int Lloc,
                       int Hq, int Hkv, int d, const int32_t* topk_idx, int k, int idx_ld,
                       const int64_t* doc_chunk_off, int64_t D, int64_t C, const void* Kbar, const void* Vbar,
                       int Mmax, float scale, void* O, float* lse, const IndexedWs& w, int32_t* err_flag,
                       cudaStream_t s) {
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d);
  AttnArgs a{Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, nullptr, nullptr, w.mem_len, Mmax, scale, O, lse,
             nullptr, 0, err_flag, nullptr, nullptr, nullptr, 0, C};
  const bool on_device = !host_resident(Kbar) && !host_resident(Vbar);
  if (on_device && C > 0 && attn_indexed_applies(dt, a)) {
    PlanArgs pa{topk_idx, B, k, doc_chunk_off, D, C, Mmax, w.Smax, w.seg_row, w.seg_cnt, w.nseg, w.mem_len, err_flag,
                idx_ld};
    if (launch_plan(pa, s) != cudaSuccess) return MSA_ERR_CUDA;
    a.Kmem = Kbar;
    a.Vmem = Vbar;
    a.seg_row = w.seg_row;
    a.seg_cnt = w.seg_cnt;
    a.nseg = w.nseg;
    a.Smax = w.Smax;
    a.ws = w.attn_ws;
    a.ws_bytes = w.attn_ws_bytes;
    return cuda_status(launch_attn(dt, a, s));
  }
  GatherArgs ga{topk_idx, B, k, doc_chunk_off, D, C, Kbar, Vbar, Hkv, d, Mmax, w.Kmem, w.Vmem, w.mem_len, err_flag,
                host_resident(Kbar), idx_ld};
  if (launch_gather(dt, ga, s) != cudaSuccess) return MSA_ERR_CUDA;
  a.Kmem = w.Kmem;
  a.Vmem = w.Vmem;
  a.ws = w.dense_ws;
  a.ws_bytes = w.dense_ws_bytes;
  return cuda_status(launch_attn(dt, a, s));
}

}  // namespace

namespace msa {
msa_status route_topk_args_status(msa_dtype dt, const void* Qr, int64_t B, int Tq, int Hr, int dr,
                                  const void* Krbar, const float* kr_rnorm, const int64_t* doc_chunk_off,
                                  int64_t D, int64_t C, int k, const int32_t* topk_idx) {
  return check_route(dt, Qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, k, topk_idx);
}
}  // namespace msa

extern "C" {

const char* msa_status_string(int status) {
  switch (status) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MSA_ERR_WORKSPACE: return "workspace missing or too small";
    case MSA_ERR_CUDA: return "CUDA launch or runtime error";
    case MSA_ERR_TOO_LARGE: return "problem larger than the no-allocation entry point's fixed scratch";
    default: return "unknown status";
  }
}

const char* msa_version(void) { return "0.1.0"; }

uint64_t msa_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void msa_testing_set_wait_polls(int64_t polls) { attn_tc_set_test_polls(polls); }

msa_status msa_rope_table_host(double theta, int d, int max_len, float* host_out) {
  if (!host_out || d < 2 || (d & 1) || max_len < 1 || !(theta > 0.0)) return MSA_ERR_INVALID_ARG;
  const int half = d / 2;
  for (int p = 0; p < max_len; ++p) {
    for (int i = 0; i < half; ++i) {
      const double ang = (double)p * pow(theta, -2.0 * (double)i / (double)d);
      host_out[((size_t)p * half + i) * 2] = (float)cos(ang);
      host_out[((size_t)p * half + i) * 2 + 1] = (float)sin(ang);
    }
  }
  return MSA_OK;
}

msa_status msa_chunk_offsets_host(const int64_t* doc_tok_off, int64_t D, int P, int64_t* out) {
  if (!doc_tok_off || !out || D < 0 || P < 1) return MSA_ERR_INVALID_ARG;
  out[0] = 0;
  for (int64_t j = 0; j < D; ++j) {
    const int64_t L = doc_tok_off[j + 1] - doc_tok_off[j];
    if (L < 0) return MSA_ERR_INVALID_ARG;
    out[j + 1] = out[j] + (L + P - 1) / P;
  }
  return MSA_OK;
}

msa_status msa_pool(msa_dtype dt, const void* K, const void* V, const void* Kr, const int64_t* doc_tok_off,
                    const int64_t* doc_chunk_off, int64_t D, int64_t Ntok, int64_t C, int Hkv, int d, int Hr,
                    int dr, int P, const float* rope_cs, int max_len, void* Kbar, void* Vbar, void* Krbar,
                    float* kr_rnorm, int32_t* err_flag, msa_stream_t stream) {
  if (!dtype_ok(dt) || D < 0 || Ntok < 0 || C < 0 || Hkv < 1 || Hr < 1 || P < 1 || max_len < 1)
    return MSA_ERR_INVALID_ARG;
  if (!head_dim_ok(d) || !head_dim_ok(dr) || P > 4096 || Hkv > 64 || Hr > 64) return MSA_ERR_UNSUPPORTED;
  if (C > kMaxIndex || D > kMaxIndex) return MSA_ERR_INVALID_ARG;
  if (C == 0) return MSA_OK;
  if (!K || !V || !Kr || !doc_tok_off || !doc_chunk_off || !rope_cs || !Kbar || !Vbar || !Krbar)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(Kr) || !aligned16(rope_cs) || !aligned16(Kbar) ||
      !aligned16(Vbar) || !aligned16(Krbar))
    return MSA_ERR_INVALID_ARG;
  // one CTA thread per 16-byte column vector must fit in a block
  const int vn = dt == MSA_F32 ? 4 : 8;
  if (Hkv * (d / 2) / vn + Hkv * d / vn + Hr * dr / vn > 480) return MSA_ERR_UNSUPPORTED;
  PoolArgs a{K, V, Kr, doc_tok_off, doc_chunk_off, D, Ntok, C, Hkv, d, Hr, dr, P, rope_cs, max_len,
             Kbar, Vbar, Krbar, kr_rnorm, err_flag};
  return cuda_status(launch_pool(dt, a, reinterpret_cast<cudaStream_t>(stream)));
}

msa_status msa_bank_rnorm(msa_dtype dt, const void* Krbar, int64_t C, int Hr, int dr, float* kr_rnorm,
                          msa_stream_t stream) {
  if (!dtype_ok(dt) || C < 0 || Hr < 1) return MSA_ERR_INVALID_ARG;
  if (!head_dim_ok(dr)) return MSA_ERR_UNSUPPORTED;
  if (C == 0) return MSA_OK;
  if (!Krbar || !kr_rnorm) return MSA_ERR_INVALID_ARG;
  return cuda_status(launch_bank_rnorm(dt, Krbar, C, Hr, dr, kr_rnorm, reinterpret_cast<cudaStream_t>(stream)));
}

size_t msa_route_topk_workspace_size(int64_t B, int Tq, int Hr, int64_t D, int64_t C, int k) {
  if (B < 0 || Tq < 1 || Hr < 1 || D < 1 || C < 0 || k < 1) return 0;
  return route_ws_layout(nullptr, B, Tq, Hr, D, C, k).bytes;
}

msa_status msa_route_topk(msa_dtype dt, const void* Qr, int64_t B, int Tq, int Hr, int dr, const void* Krbar,
                          const float* kr_rnorm, const int64_t* doc_chunk_off, int64_t D, int64_t C, int k,
                          float* doc_scores, int32_t* topk_idx, float* topk_score, void* ws, size_t ws_bytes,
                          int32_t* err_flag, msa_stream_t stream) {
  msa_status st = check_route(dt, Qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, k, topk_idx);
  if (st != MSA_OK) return st;
  if (B == 0) return MSA_OK;
  RouteWs w = route_ws_layout(ws, B, Tq, Hr, D, C, k);
  if (!ws || ws_bytes < w.bytes || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  RouteArgs ra{Qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, w.doc_key, w.rq, w.chunk_doc, err_flag};
  cudaError_t e = launch_route(dt, ra, s);
  if (e != cudaSuccess) return MSA_ERR_CUDA;
  TopkArgs ta{w.doc_key, B, D, k, w.cand, w.doc_key + B * D, w.nslice, topk_idx, topk_score, doc_scores};
  return cuda_status(launch_topk(ta, s));
}

msa_status msa_gather(msa_dtype dt, const int32_t* topk_idx, int64_t B, int k, const int64_t* doc_chunk_off,
                      int64_t D, int64_t C, const void* Kbar, const void* Vbar, int Hkv, int d, int Mmax,
                      void* Kmem, void* Vmem, int32_t* mem_len, int32_t* err_flag, msa_stream_t stream) {
  if (!dtype_ok(dt) || B < 0 || k < 1 || D < 1 || C < 0 || Hkv < 1 || Mmax < 0) return MSA_ERR_INVALID_ARG;
  if (!head_dim_ok(d) || B > 65535 || k > 65535) return MSA_ERR_UNSUPPORTED;
  if (B == 0) return MSA_OK;
  if (!topk_idx || !doc_chunk_off || !Kbar || !Vbar || !mem_len || (Mmax > 0 && (!Kmem || !Vmem)))
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(Kbar) || !aligned16(Vbar) || !aligned16(Kmem) || !aligned16(Vmem)) return MSA_ERR_INVALID_ARG;
  if (!device_readable(Kbar) || !device_readable(Vbar)) return MSA_ERR_INVALID_ARG;
  GatherArgs a{topk_idx, B, k, doc_chunk_off, D, C, Kbar, Vbar, Hkv, d, Mmax, Kmem, Vmem, mem_len, err_flag,
               host_resident(Kbar)};
  return cuda_status(launch_gather(dt, a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t msa_sparse_attn_backward_workspace_size(int64_t B, int Tq, int Hq) {
  if (B < 0 || Tq < 1 || Hq < 1) return 0;
  return attn_bwd_workspace_size(B, Tq, Hq);
}

msa_status msa_sparse_attn_backward(msa_dtype dt, const void* Q, const void* Kloc, const void* Vloc, int64_t B,
                                    int Tq, int Lloc, int Hq, int Hkv, int d, const void* Kmem, const void* Vmem,
                                    const int32_t* mem_len, int Mmax, float scale, const void* O, const float* lse,
                                    const void* dO, float* dQ, float* dKloc, float* dVloc, float* dKmem,
                                    float* dVmem, void* ws, size_t ws_bytes, int32_t* err_flag,
                                    msa_stream_t stream) {
  msa_status st = check_attn(dt, Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, Mmax);
  if (st != MSA_OK) return st;
  if (B == 0) return MSA_OK;
  if (!mem_len || !O || !lse || !dO || !dQ || !dKloc || !dVloc) return MSA_ERR_INVALID_ARG;
  if (Mmax > 0 && (!Kmem || !Vmem || !dKmem || !dVmem)) return MSA_ERR_INVALID_ARG;
  if (!aligned16(O) || !aligned16(dO) || !aligned16(Kmem) || !aligned16(Vmem)) return MSA_ERR_INVALID_ARG;
  const size_t need = attn_bwd_workspace_size(B, Tq, Hq);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  AttnBwdArgs a{Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, Kmem, Vmem, mem_len, Mmax,
                scale > 0.f ? scale : 1.0f / sqrtf((float)d), O, dO, lse, dQ, dKloc, dVloc, dKmem, dVmem,
                static_cast<float*>(ws), err_flag};
  return cuda_status(launch_attn_bwd(dt, a, reinterpret_cast<cudaStream_t>(stream)));
}

msa_status msa_gather_backward(const int32_t* topk_idx, int64_t B, int k, const int64_t* doc_chunk_off, int64_t D,
                               int64_t C, const float* dKmem, const float* dVmem, const int32_t* mem_len, int Hkv,
                               int d, int Mmax, float* dKbar, float* dVbar, int32_t* err_flag,
                               msa_stream_t stream) {
  if (B < 0 || k < 1 || D < 1 || C < 0 || Hkv < 1 || Mmax < 0) return MSA_ERR_INVALID_ARG;
  if (!head_dim_ok(d) || B > 65535 || k > 65535) return MSA_ERR_UNSUPPORTED;
  if (B == 0 || Mmax == 0) return MSA_OK;
  if (!topk_idx || !doc_chunk_off || !dKmem || !dVmem || !mem_len || !dKbar || !dVbar) return MSA_ERR_INVALID_ARG;
  GatherBwdArgs a{topk_idx, B, k, doc_chunk_off, D, C, dKmem, dVmem, mem_len, Hkv, d, Mmax, dKbar, dVbar, err_flag};
  return cuda_status(launch_gather_bwd(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t msa_route_backward_workspace_size(int64_t B, int Tq, int k) {
  if (B < 0 || Tq < 1 || k < 1) return 0;
  return route_bwd_workspace_size(B, Tq, k);
}

msa_status msa_route_backward(msa_dtype dt, const void* Qr, int64_t B, int Tq, int Hr, int dr, const void* Krbar,
                              const float* kr_rnorm, const int64_t* doc_chunk_off, int64_t D, int64_t C, int k,
                              const int32_t* topk_idx, const float* d_score, float* dQr, float* dKrbar, void* ws,
                              size_t ws_bytes, int32_t* err_flag, msa_stream_t stream) {
  msa_status st = check_route(dt, Qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, k, topk_idx);
  if (st != MSA_OK) return st;
  if (B > 65535 || k > 65535) return MSA_ERR_UNSUPPORTED;
  if (B == 0) return MSA_OK;
  if (!d_score || !dQr || !dKrbar) return MSA_ERR_INVALID_ARG;
  const size_t need = route_bwd_workspace_size(B, Tq, k);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  RouteBwdArgs a{Qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, k, topk_idx, d_score,
                 dQr, dKrbar, ws, err_flag};
  return cuda_status(launch_route_bwd(dt, a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t msa_sparse_attn_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, int Mmax) {
  return attn_workspace_size(MSA_BF16, B, Tq, Lloc, Hq, Hkv, d, Mmax);
}

msa_status msa_sparse_attn(msa_dtype dt, const void* Q, const void* Kloc, const void* Vloc, int64_t B, int Tq,
                           int Lloc, int Hq, int Hkv, int d, const void* Kmem, const void* Vmem,
                           const int32_t* mem_len, int Mmax, float scale, void* O, float* lse, void* ws,
                           size_t ws_bytes, int32_t* err_flag, msa_stream_t stream) {
  msa_status st = check_attn(dt, Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, Mmax);
  if (st != MSA_OK) return st;
  if (B == 0) return MSA_OK;
  if (!O || !mem_len || (Mmax > 0 && (!Kmem || !Vmem))) return MSA_ERR_INVALID_ARG;
  if (!aligned16(O) || !aligned16(Kmem) || !aligned16(Vmem)) return MSA_ERR_INVALID_ARG;
  const size_t need = attn_workspace_size(dt, B, Tq, Lloc, Hq, Hkv, d, Mmax);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return MSA_ERR_WORKSPACE;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d);
  AttnArgs a{Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, Kmem, Vmem, mem_len, Mmax, scale, O, lse,
             ws, ws_bytes, err_flag};
  return cuda_status(launch_attn(dt, a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t msa_sparse_attn_indexed_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, int k,
                                              int Mmax) {
  if (B < 0 || Tq < 1 || Lloc < 1 || Hq < 1 || Hkv < 1 || d < 1 || k < 1 || Mmax < 0) return 0;
  return indexed_ws_layout(nullptr, B, Tq, Lloc, Hq, Hkv, d, k, Mmax).bytes;
}

msa_status msa_sparse_attn_indexed(msa_dtype dt, const void* Q, const void* Kloc, const void* Vloc, int64_t B,
                                   int Tq, int Lloc, int Hq, int Hkv, int d, const int32_t* topk_idx, int k,
                                   const int64_t* doc_chunk_off, int64_t D, int64_t C, const void* Kbar,
                                   const void* Vbar, int Mmax, float scale, void* O, float* lse, void* ws,
                                   size_t ws_bytes, int32_t* err_flag, msa_stream_t stream) {
  msa_status st = check_attn(dt, Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, Mmax);
  if (st != MSA_OK) return st;
  st = check_indexed(topk_idx, k, doc_chunk_off, D, C, Kbar, Vbar);
  if (st != MSA_OK) return st;
  if (B == 0) return MSA_OK;
  if (!O || !aligned16(O)) return MSA_ERR_INVALID_ARG;
  const IndexedWs w = indexed_ws_layout(ws, B, Tq, Lloc, Hq, Hkv, d, k, Mmax);
  if (!ws || ws_bytes < w.bytes || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  if (!device_readable(Kbar) || !device_readable(Vbar)) return MSA_ERR_INVALID_ARG;
  return run_indexed(dt, Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, topk_idx, k, k, doc_chunk_off, D, C, Kbar, Vbar,
                     Mmax, scale, O, lse, w, err_flag, reinterpret_cast<cudaStream_t>(stream));
}

size_t msa_layer_forward_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, int Hr, int64_t D,
                                        int64_t C, int k, int Mmax) {
  if (B < 0 || Tq < 1 || Lloc < 1 || Hq < 1 || Hkv < 1 || d < 1 || Hr < 1 || D < 1 || C < 0 || k < 1 || Mmax < 0)
    return 0;
  return route_ws_layout(nullptr, B, Tq, Hr, D, C, k).bytes +
         indexed_ws_layout(nullptr, B, Tq, Lloc, Hq, Hkv, d, k, Mmax).bytes;
}

msa_status msa_layer_forward(msa_dtype dt, const void* Qr, int Hr, int dr, const void* Krbar,
                             const float* kr_rnorm, const int64_t* doc_chunk_off, int64_t D, int64_t C, int k,
                             const void* Q, const void* Kloc, const void* Vloc, int64_t B, int Tq, int Lloc,
                             int Hq, int Hkv, int d, const void* Kbar, const void* Vbar, int Mmax, float scale,
                             void* O, float* lse, int32_t* topk_idx, float* topk_score, float* doc_scores,
                             void* ws, size_t ws_bytes, int32_t* err_flag, msa_stream_t stream) {
  msa_status st = check_route(dt, Qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, k, topk_idx);
  if (st != MSA_OK) return st;
  st = check_attn(dt, Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, Mmax);
  if (st != MSA_OK) return st;
  st = check_indexed(topk_idx, k, doc_chunk_off, D, C, Kbar, Vbar);
  if (st != MSA_OK) return st;
  if (B == 0) return MSA_OK;
  if (!O || !aligned16(O)) return MSA_ERR_INVALID_ARG;
  const size_t need = msa_layer_forward_workspace_size(B, Tq, Lloc, Hq, Hkv, d, Hr, D, C, k, Mmax);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  if (!device_readable(Kbar) || !device_readable(Vbar)) return MSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  RouteWs w = route_ws_layout(ws, B, Tq, Hr, D, C, k);
  const IndexedWs iw = indexed_ws_layout(static_cast<char*>(ws) + w.bytes, B, Tq, Lloc, Hq, Hkv, d, k, Mmax);
  RouteArgs ra{Qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, w.doc_key, w.rq, w.chunk_doc, err_flag};
  if (launch_route(dt, ra, s) != cudaSuccess) return MSA_ERR_CUDA;
  TopkArgs ta{w.doc_key, B, D, k, w.cand, w.doc_key + B * D, w.nslice, topk_idx, topk_score, doc_scores};
  if (launch_topk(ta, s) != cudaSuccess) return MSA_ERR_CUDA;
  return run_indexed(dt, Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, topk_idx, k, k, doc_chunk_off, D, C, Kbar, Vbar,
                     Mmax, scale, O, lse, iw, err_flag, s);
}

size_t msa_interleave_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, int Hr, int dr, int64_t D,
                                     int64_t C, int k, int rounds, int Mmax) {
  if (B < 0 || Tq < 1 || Lloc < 1 || Hq < 1 || Hkv < 1 || d < 1 || Hr < 1 || dr < 1 || D < 1 || C < 0 || k < 1 ||
      rounds < 1 || Mmax < 0 || (int64_t)rounds * k > kMaxIndex)
    return 0;
  return route_ws_layout(nullptr, B, Tq, Hr, D, C, k).bytes +
         indexed_ws_layout(nullptr, B, Tq, Lloc, Hq, Hkv, d, rounds * k, Mmax).bytes +
         round_up(sizeof(float) * (size_t)B * (size_t)Tq * (size_t)Hr * (size_t)dr, 256);
}

msa_status msa_interleave_forward(msa_dtype dt, const void* Qr0, int Hr, int dr, const void* Krbar,
                                  const float* kr_rnorm, const int64_t* doc_chunk_off, int64_t D, int64_t C, int k,
                                  int rounds, const void* W_route, const void* Q, const void* Kloc, const void* Vloc,
                                  int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, const void* Kbar,
                                  const void* Vbar, int Mmax, float scale, void* O, float* lse, void* O_rounds,
                                  void* Qr_rounds, int32_t* topk_idx, float* topk_score, void* ws, size_t ws_bytes,
                                  int32_t* err_flag, msa_stream_t stream) {
  if (rounds < 1 || k < 1 || (int64_t)rounds * k > D) return MSA_ERR_INVALID_ARG;
  msa_status st = check_route(dt, Qr0, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, k, topk_idx);
  if (st != MSA_OK) return st;
  st = check_attn(dt, Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, Mmax);
  if (st != MSA_OK) return st;
  st = check_indexed(topk_idx, rounds * k, doc_chunk_off, D, C, Kbar, Vbar);
  if (st != MSA_OK) return st;
  if (rounds > 1 && !W_route) return MSA_ERR_INVALID_ARG;
  if (B * (int64_t)Tq > 65535ll * 16) return MSA_ERR_UNSUPPORTED;  // rows of the round-to-round map's grid
  if (B == 0) return MSA_OK;
  if (!O || !aligned16(O) || !aligned16(O_rounds) || !aligned16(Qr_rounds)) return MSA_ERR_INVALID_ARG;
  const size_t need = msa_interleave_workspace_size(B, Tq, Lloc, Hq, Hkv, d, Hr, dr, D, C, k, rounds, Mmax);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  if (!device_readable(Kbar) || !device_readable(Vbar)) return MSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const RouteWs w = route_ws_layout(ws, B, Tq, Hr, D, C, k);
  char* p = static_cast<char*>(ws) + w.bytes;
  const IndexedWs iw = indexed_ws_layout(p, B, Tq, Lloc, Hq, Hkv, d, rounds * k, Mmax);
  void* qr_ws = p + iw.bytes;
  const int ld = rounds * k;
  const size_t esz = dt == MSA_F32 ? 4 : 2;
  const size_t o_bytes = (size_t)B * Tq * Hq * d * esz;
  const size_t qr_bytes = (size_t)B * Tq * Hr * dr * esz;
  // round r >= 1 routes with the router query the map wrote: slot r - 1 of Qr_rounds, or the workspace
  auto qr_slot = [&](int r) -> void* {
    return Qr_rounds ? static_cast<char*>(Qr_rounds) + (size_t)(r - 1) * qr_bytes : qr_ws;
  };
  for (int r = 0; r < rounds; ++r) {
    const void* qr = r == 0 ? Qr0 : qr_slot(r);
    RouteArgs ra{qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, w.doc_key, w.rq, w.chunk_doc, err_flag};
    if (launch_route(dt, ra, s) != cudaSuccess) return MSA_ERR_CUDA;
    // documents of the earlier rounds are passed over
    if (launch_exclude(w.doc_key, B, D, topk_idx, ld, r * k, s) != cudaSuccess) return MSA_ERR_CUDA;
    TopkArgs ta{w.doc_key, B, D, k, w.cand, w.doc_key + B * D, w.nslice, topk_idx + (size_t)r * k,
                topk_score ? topk_score + (size_t)r * k : nullptr, nullptr, ld};
    if (launch_topk(ta, s) != cudaSuccess) return MSA_ERR_CUDA;
    const bool last = r == rounds - 1;
    void* Or = (last || !O_rounds) ? O : static_cast<char*>(O_rounds) + (size_t)r * o_bytes;
    st = run_indexed(dt, Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, topk_idx, (r + 1) * k, ld, doc_chunk_off, D, C,
                     Kbar, Vbar, Mmax, scale, Or, last ? lse : nullptr, iw, err_flag, s);
    if (st != MSA_OK) return st;
    if (!last && launch_project(dt, Or, W_route, qr_slot(r + 1), B * (int64_t)Tq, Hq * d, Hr * dr, s) != cudaSuccess)
      return MSA_ERR_CUDA;
  }
  return MSA_OK;
}

msa_status msa_gated_delta_rule(msa_dtype dt, const void* q, const void* k, const void* v, const float* g,
                                const float* beta, int64_t B, int T, int Hk, int Hv, int dk, int dv, const float* h0,
                                float scale, void* o, float* hT, msa_stream_t stream) {
  if (!dtype_ok(dt) || B < 0 || T < 0 || Hk < 1 || Hv < 1 || Hv % Hk != 0) return MSA_ERR_INVALID_ARG;
  if (dk != 128 || dv != 128 || B > 65535 || Hv > 65535) return MSA_ERR_UNSUPPORTED;
  if (B == 0 || T == 0) return MSA_OK;
  if (!q || !k || !v || !g || !beta || !o) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return MSA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)dk);
  return cuda_status(launch_gdr(dt, q, k, v, g, beta, B, T, Hk, Hv, dk, h0, scale, o, hT,
                                reinterpret_cast<cudaStream_t>(stream)));
}

msa_status msa_state_gather_sum(msa_dtype dt, const void* states, int64_t D, int64_t S, const int32_t* topk_idx,
                                int64_t B, int k, float* S_ext, int32_t* err_flag, msa_stream_t stream) {
  if (!dtype_ok(dt) || D < 1 || S < 1 || B < 0 || k < 1) return MSA_ERR_INVALID_ARG;
  if (S % (dt == MSA_F32 ? 4 : 8) != 0 || B > 65535) return MSA_ERR_UNSUPPORTED;  // 16-byte vectors
  if (B == 0) return MSA_OK;
  if (!states || !topk_idx || !S_ext) return MSA_ERR_INVALID_ARG;
  if (!aligned16(states) || !aligned16(S_ext) || !device_readable(states)) return MSA_ERR_INVALID_ARG;
  return cuda_status(launch_state_sum(dt, states, D, S, topk_idx, B, k, S_ext, err_flag,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
