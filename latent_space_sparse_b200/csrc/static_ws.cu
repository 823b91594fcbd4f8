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
#include "common.cuh"

namespace {

// Scratch of salsc_decode_step_static_ws.  Every GPU that loads this part of
// the library holds SALSC_STATIC_WORKSPACE_BYTES for it until the process
// exits.  All calls on a device share it and it keeps the last call's
// contents.
static __device__ __align__(256) unsigned char g_static_ws[SALSC_STATIC_WORKSPACE_BYTES];

// Device address of g_static_ws on the current device.  Host code cannot use
// the symbol itself (on the host it names a stand-in, not device memory), so
// every call asks the runtime for the address with the caller's device
// current.  The first call on a device loads the array's module; later
// lookups are cheap, and a device reset between calls leaves no stale
// address behind.
salsc_status static_ws_address(void** addr) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_static_ws);
  if (e != cudaSuccess) return salsc::record_cuda_error(e);
  *addr = p;
  return SALSC_OK;
}

}  // namespace

extern "C" size_t salsc_static_workspace_bytes(void) { return SALSC_STATIC_WORKSPACE_BYTES; }

extern "C" salsc_status salsc_decode_step_static_ws(const salsc_decode_desc* desc, const void* q,
                                                   const void* Kc, const void* Vc, const void* Pk,
                                                   const void* Pv, void* out, int32_t* idx_out,
                                                   salsc_stream stream) {
  // every argument is checked first: a rejected call enqueues nothing
  salsc_status st = salsc::check_decode_step(desc, q, Kc, Vc, Pk, Pv, out, idx_out);
  if (st != SALSC_OK) return st;
  if (salsc_decode_workspace_size(desc) > (size_t)SALSC_STATIC_WORKSPACE_BYTES)
    return SALSC_ERR_WORKSPACE;
  void* ws = nullptr;
  if ((st = static_ws_address(&ws)) != SALSC_OK) return st;
  // The array keeps the previous call's contents: the anomaly word (the only
  // part that must start at zero) is cleared on the same stream, once every
  // argument has been checked.
  return salsc::decode_step_clearing_flags(desc, q, Kc, Vc, Pk, Pv, out, idx_out, ws,
                                           SALSC_STATIC_WORKSPACE_BYTES, stream);
}
