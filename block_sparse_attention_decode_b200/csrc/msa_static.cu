// msa_static.cu -- msa_decode_static: the whole decode step with its
// scratch in a fixed, library-owned device array instead of a caller-provided
// workspace.  The method's pages have no counterpart for this entry point; it
// exists for callers that cannot allocate device memory on the calling path.
//
// The scratch is a file-scope __device__ array of MSA_STATIC_WORKSPACE_BYTES.
// In host code its name is only a host-side stand-in, never a device
// address: the device address is fetched with cudaGetSymbolAddress (with the
// device current) at set-up, once per device, and cached together with the
// identity of the device's CUDA context.  If that context is no longer the
// current one (a cudaDeviceReset destroyed it and a new one was created), the
// set-up runs again, so the cached address is never used in a context it does
// not belong to.  Each call clears the part that must start at zero (the
// error flags; the split-K counters are cleared by the attention launch
// itself) and then runs the same kernels as msa_decode on that memory.
#include <cuda.h>

#include <mutex>

#include "msa.h"
#include "msa_internal.h"

namespace {

__device__ __align__(256) uint8_t g_static_ws[MSA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ws_ptr[kMaxDevices] = {};
unsigned long long g_ws_ctx[kMaxDevices] = {};   // context id the address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the current CUDA context (ids are never reused in a process).
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (get_current == nullptr || get_id == nullptr) {
    void* p0 = nullptr;
    void* p1 = nullptr;
    cudaDriverEntryPointQueryResult q0{}, q1{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p0, cudaEnableDefault, &q0) != cudaSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &p1, cudaEnableDefault, &q1) != cudaSuccess ||
        q0 != cudaDriverEntryPointSuccess || q1 != cudaDriverEntryPointSuccess || !p0 || !p1) {
      cudaGetLastError();
      return false;
    }
    get_current = reinterpret_cast<CtxGetCurrentFn>(p0);
    get_id = reinterpret_cast<CtxGetIdFn>(p1);
  }
  CUcontext ctx = nullptr;
  return get_current(&ctx) == CUDA_SUCCESS && ctx != nullptr && get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_static_ws on the current device (set-up on first use
// in the device's current context).
msa_status static_workspace(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return MSA_ERR_CUDA; }
  if (dev < 0 || dev >= kMaxDevices) return MSA_ERR_UNSUPPORTED;
  // makes the device's primary context current (created again if a reset
  // destroyed it): cudaSetDevice initialises the context since CUDA 12
  if (cudaSetDevice(dev) != cudaSuccess) { cudaGetLastError(); return MSA_ERR_CUDA; }
  unsigned long long ctx = 0;
  if (!current_context_id(&ctx)) return MSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_ws_ptr[dev] == nullptr || g_ws_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MSA_ERR_CUDA;
    }
    g_ws_ptr[dev] = p;
    g_ws_ctx[dev] = ctx;
  }
  *ptr = g_ws_ptr[dev];
  return MSA_OK;
}

}  // namespace

extern "C" MSA_API msa_status msa_decode_static(const msa_cache* cache, const msa_seqs* seqs,
                                                const uint8_t* qi, float s_qi, const uint8_t* q,
                                                float s_q, float softmax_scale, uint16_t* out,
                                                int32_t* sel_out, msa_stream_t stream) {
  const size_t need = msa::workspace_base_size(seqs);   // decode-once rows only if they fit too
  if (need == 0) return MSA_ERR_INVALID_ARG;
  if (need > (size_t)MSA_STATIC_WORKSPACE_BYTES) return MSA_ERR_WORKSPACE;
  void* ws = nullptr;
  msa_status st = static_workspace(&ws);
  if (st != MSA_OK) return st;
  // the error flags (first 256 bytes) must start at zero for every call
  if (cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return MSA_ERR_CUDA;
  }
  return msa_decode(cache, seqs, qi, s_qi, q, s_q, softmax_scale, out, sel_out, ws,
                    (size_t)MSA_STATIC_WORKSPACE_BYTES, stream);
}
