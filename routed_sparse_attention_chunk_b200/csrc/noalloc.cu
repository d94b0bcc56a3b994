// msa_route_topk_noalloc: routing + top-k with library-owned scratch memory.
//
// Some callers cannot hand the library a workspace: a plugin inside a host
// framework whose allocator owns all device memory and offers it no scratch,
// or a serving loop that must not allocate once it is running, because an
// allocation can block on the device or fail under memory pressure.  For them
// this entry point takes its scratch from a fixed array in the library's own
// device memory instead of from the caller.
//
// The array is a file-scope __device__ variable of kScratchBytes; every GPU
// that loads the library holds it until the process exits.  Host code cannot
// use the array's name as a device address (in host code it is only a
// stand-in), so the first call on each device, with that device current,
// looks the address up with cudaGetSymbolAddress and caches it.  That first
// call should therefore happen before any stream capture.  All calls share the
// one array and it keeps the previous call's contents: the routing launcher
// zeroes the per-document maxima before it uses them and every other part is
// written before it is read.  Calls that overlap on the GPU (for example on two
// streams at once) race on the array and must not be issued.
#include <mutex>

#include "internal.h"
#include "msa.h"

namespace {

constexpr size_t kScratchBytes = (size_t)MSA_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once).
msa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return MSA_ERR_CUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return MSA_OK;
}

}  // namespace

extern "C" msa_status msa_route_topk_noalloc(msa_dtype dt, const void* Qr, int64_t B, int Tq, int Hr, int dr,
                                             const void* Krbar, const float* kr_rnorm,
                                             const int64_t* doc_chunk_off, int64_t D, int64_t C, int k,
                                             float* doc_scores, int32_t* topk_idx, float* topk_score,
                                             int32_t* err_flag, msa_stream_t stream) {
  if (B < 0 || Tq < 1 || Hr < 1 || D < 1 || C < 0 || k < 1) return MSA_ERR_INVALID_ARG;
  if (B == 0) return MSA_OK;
  const size_t need = msa_route_topk_workspace_size(B, Tq, Hr, D, C, k);
  if (need == 0 || need > kScratchBytes) return MSA_ERR_TOO_LARGE;
  void* ws = nullptr;
  const msa_status st = scratch_address(&ws);
  if (st != MSA_OK) return st;
  return msa_route_topk(dt, Qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, k, doc_scores, topk_idx,
                        topk_score, ws, kScratchBytes, err_flag, stream);
}
