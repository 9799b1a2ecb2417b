// msa_static.cu -- msa_decode_static: the whole decode step with its
// scratch in a fixed, library-owned device array instead of a caller-provided
// workspace.  The method's pages have no counterpart for this entry point; it
// exists for callers that cannot allocate device memory on the calling path.
//
// The scratch is a file-scope __device__ array of MSA_STATIC_WORKSPACE_BYTES.
// In host code its name is only a host-side stand-in, never a device
// address: the device address is fetched once per device with
// cudaGetSymbolAddress (with that device current) and cached.  Each call
// clears the part that must start at zero (the error flags; the split-K
// counters are cleared by the attention launch itself) and then runs the same
// kernels as msa_decode on that memory.
#include <mutex>

#include "msa.h"
#include "msa_internal.h"

namespace {

__device__ __align__(256) uint8_t g_static_ws[MSA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ws_ptr[kMaxDevices] = {};

// Device address of g_static_ws on the current device (set-up on first use).
msa_status static_workspace(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return MSA_ERR_CUDA; }
  if (dev < 0 || dev >= kMaxDevices) return MSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_ws_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MSA_ERR_CUDA;
    }
    g_ws_ptr[dev] = p;
  }
  *ptr = g_ws_ptr[dev];
  return MSA_OK;
}

}  // namespace

extern "C" MSA_API msa_status msa_decode_static(const msa_cache* cache, const msa_seqs* seqs,
                                                const uint8_t* qi, float s_qi, const uint8_t* q,
                                                float s_q, float softmax_scale, uint16_t* out,
                                                int32_t* sel_out, msa_stream_t stream) {
  const size_t need = msa_workspace_size(seqs);
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
