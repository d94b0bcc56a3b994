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
// looks the address up with cudaGetSymbolAddress and caches it together with
// the CUDA context it belongs to; a call from a different context on that
// device (after a device reset, say) looks it up again.  A first call should
// therefore happen before any stream capture.  All calls share the one array
// and it keeps the previous call's contents: the routing launcher zeroes the
// per-document maxima and the top-k counters before it uses them, and every
// other part is written before it is read.  Calls that overlap on the GPU (for
// example on two streams at once) race on the array and must not be issued.
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"
#include "msa.h"

namespace {

constexpr size_t kScratchBytes = (size_t)MSA_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct Cached {
  CUcontext ctx;
  void* addr;
};
Cached g_cache[kMaxDevices] = {};

// cuCtxGetCurrent through the runtime's driver entry point (the library does not link libcuda).
PFN_cuCtxGetCurrent_v4000 ctx_get_current() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  return fn;
}

// Device address of the scratch array in the current device's current context.
msa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MSA_ERR_CUDA;
  auto get = ctx_get_current();
  CUcontext ctx = nullptr;
  if (!get || get(&ctx) != CUDA_SUCCESS) return MSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  Cached& c = g_cache[dev];
  if (!ctx || c.ctx != ctx || !c.addr) {
    // the lookup also makes the runtime's context for the device current when none was yet
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return MSA_ERR_CUDA;
    if (get(&ctx) != CUDA_SUCCESS || !ctx) return MSA_ERR_CUDA;
    c.ctx = ctx;
    c.addr = p;
  }
  *out = c.addr;
  return MSA_OK;
}

}  // namespace

extern "C" msa_status msa_route_topk_noalloc(msa_dtype dt, const void* Qr, int64_t B, int Tq, int Hr, int dr,
                                             const void* Krbar, const float* kr_rnorm,
                                             const int64_t* doc_chunk_off, int64_t D, int64_t C, int k,
                                             float* doc_scores, int32_t* topk_idx, float* topk_score,
                                             int32_t* err_flag, msa_stream_t stream) {
  // the same argument errors, in the same order, as msa_route_topk; then the size check
  const msa_status chk =
      msa::route_topk_args_status(dt, Qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, k, topk_idx);
  if (chk != MSA_OK) return chk;
  if (B == 0) return MSA_OK;
  if (msa_route_topk_workspace_size(B, Tq, Hr, D, C, k) > kScratchBytes) return MSA_ERR_TOO_LARGE;
  void* ws = nullptr;
  const msa_status st = scratch_address(&ws);
  if (st != MSA_OK) return st;
  return msa_route_topk(dt, Qr, B, Tq, Hr, dr, Krbar, kr_rnorm, doc_chunk_off, D, C, k, doc_scores, topk_idx,
                        topk_score, ws, kScratchBytes, err_flag, stream);
}
