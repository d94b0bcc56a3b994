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

size_t msa_layer_forward_workspace_size(int64_t B, int Tq, int Lloc, int Hq, int Hkv, int d, int Hr, int64_t D,
                                        int64_t C, int k, int Mmax) {
  if (B < 0 || Tq < 1 || Hr < 1 || D < 1 || C < 0 || k < 1 || Mmax < 0) return 0;
  size_t n = route_ws_layout(nullptr, B, Tq, Hr, D, C, k).bytes;
  // gathered memory rows (sized for fp32 storage, the larger type) and their counts
  n += 2 * round_up(sizeof(float) * (size_t)B * (size_t)Mmax * (size_t)Hkv * (size_t)d, 256);
  n += round_up(sizeof(int32_t) * (size_t)B, 256);
  n += round_up(attn_workspace_size(MSA_BF16, B, Tq, Lloc, Hq, Hkv, d, Mmax), 256);
  return n;
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
  if (B == 0) return MSA_OK;
  if (!O || !Kbar || !Vbar || !aligned16(O) || !aligned16(Kbar) || !aligned16(Vbar)) return MSA_ERR_INVALID_ARG;
  const size_t need = msa_layer_forward_workspace_size(B, Tq, Lloc, Hq, Hkv, d, Hr, D, C, k, Mmax);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  if (!device_readable(Kbar) || !device_readable(Vbar)) return MSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  RouteWs w = route_ws_layout(ws, B, Tq, Hr, D, C, k);
  char* p = static_cast<char*>(ws) + w.bytes;
  const size_t mem_bytes = round_up(sizeof(float) * (size_t)B * (size_t)Mmax * (size_t)Hkv * (size_t)d, 256);
  void* Kmem = p;
  void* Vmem = p + mem_bytes;
  p += 2 * mem_bytes;
  int32_t* mem_len = reinterpret_cast<int32_t*>(p);
  p += round_up(sizeof(int32_t) * (size_t)B, 256);
  void* attn_ws = p;
  const size_t attn_ws_bytes = ws_bytes - (size_t)(p - static_cast<char*>(ws));

  RouteArgs ra{Qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, w.doc_key, w.rq, w.chunk_doc, err_flag};
  if (launch_route(dt, ra, s) != cudaSuccess) return MSA_ERR_CUDA;
  TopkArgs ta{w.doc_key, B, D, k, w.cand, w.doc_key + B * D, w.nslice, topk_idx, topk_score, doc_scores};
  if (launch_topk(ta, s) != cudaSuccess) return MSA_ERR_CUDA;
  GatherArgs ga{topk_idx, B, k, doc_chunk_off, D, C, Kbar, Vbar, Hkv, d, Mmax, Kmem, Vmem, mem_len, err_flag,
                host_resident(Kbar)};
  if (launch_gather(dt, ga, s) != cudaSuccess) return MSA_ERR_CUDA;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d);
  AttnArgs a{Q, Kloc, Vloc, B, Tq, Lloc, Hq, Hkv, d, Kmem, Vmem, mem_len, Mmax, scale, O, lse,
             attn_ws, attn_ws_bytes, err_flag};
  return cuda_status(launch_attn(dt, a, s));
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
