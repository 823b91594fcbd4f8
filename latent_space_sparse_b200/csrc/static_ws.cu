// static_ws.cu -- decode entry point with library-owned scratch: the caller
// allocates nothing.
//
// The SALS paper has no counterpart to this file.  It serves callers that
// cannot allocate device memory for a workspace: for example a plugin inside
// a host application whose memory manager owns every device allocation and
// forbids side allocations, or a latency-critical serving loop that must not
// call cudaMalloc (which can synchronise the whole device).  Such callers
// still pass their inputs and outputs; the decode step's scratch (latent
// queries, scores, selected indices, split partials) lives in the
// fixed-size array below instead of a caller-supplied workspace.
#include <mutex>

#include "common.cuh"

namespace {

// Scratch of salsc_decode_step_static_ws.  Every GPU that loads this part of
// the library holds SALSC_STATIC_WORKSPACE_BYTES for it until the process
// exits.  All calls on a device share it and it keeps the last call's
// contents.
static __device__ __align__(256) unsigned char g_static_ws[SALSC_STATIC_WORKSPACE_BYTES];

std::mutex g_mu;
void* g_ws_addr[salsc::kMaxDevices] = {};

// Device address of g_static_ws on the current device.  Host code cannot use
// the symbol itself (on the host it names a stand-in, not device memory), so
// the first call on each device asks the runtime for the address, with that
// device current, and caches it.
salsc_status static_ws_address(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return salsc::record_cuda_error(e);
  if (dev < 0 || dev >= salsc::kMaxDevices) return SALSC_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ws_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_ws);
    if (e != cudaSuccess) return salsc::record_cuda_error(e);
    g_ws_addr[dev] = p;
  }
  *addr = g_ws_addr[dev];
  return SALSC_OK;
}

}  // namespace

extern "C" salsc_status salsc_decode_step_static_ws(const salsc_decode_desc* desc, const void* q,
                                                   const void* Kc, const void* Vc, const void* Pk,
                                                   const void* Pv, void* out, int32_t* idx_out,
                                                   salsc_stream stream) {
  const size_t need = salsc_decode_workspace_size(desc);
  if (need == 0)  // invalid or unsupported shape: report why, enqueue nothing
    return salsc_decode_step(desc, q, Kc, Vc, Pk, Pv, out, idx_out, nullptr, 0, stream);
  if (need > (size_t)SALSC_STATIC_WORKSPACE_BYTES) return SALSC_ERR_WORKSPACE;
  void* ws = nullptr;
  salsc_status st = static_ws_address(&ws);
  if (st != SALSC_OK) return st;
  // The array keeps the previous call's contents: clear the anomaly word
  // (the only part that must start at zero) on the same stream.
  st = salsc_decode_prepare(desc, ws, SALSC_STATIC_WORKSPACE_BYTES, stream);
  if (st != SALSC_OK) return st;
  return salsc_decode_step(desc, q, Kc, Vc, Pk, Pv, out, idx_out, ws,
                           SALSC_STATIC_WORKSPACE_BYTES, stream);
}
