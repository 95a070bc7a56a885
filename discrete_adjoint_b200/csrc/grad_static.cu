// grad_static.cu -- gs_grad_static: the gradient entry point for callers that
// cannot allocate device memory.
//
// Some callers have no way to obtain scratch memory at run time: a plugin
// inside a host application that owns and budgets all device memory, a
// real-time loop in which a cudaMalloc (which may synchronize the device) is
// forbidden, or a plain C host with no allocator of its own.  gs_grad needs a
// checkpoint workspace from its caller; this variant uses instead a
// fixed-size array that lives in this file as a device global, so the caller
// passes only its inputs and outputs.
//
// Costs and limits: every GPU that loads the library holds the array
// (GS_STATIC_SCRATCH_BYTES) until the process exits; problems whose workspace
// exceeds it are rejected; all calls share the one array, so calls that
// overlap on the GPU (different streams, or other threads) race and corrupt
// each other's results.  The array keeps the previous call's contents; the
// kernels write every checkpoint before they read it, so nothing needs to be
// cleared between calls.
//
// The paper has no counterpart for this entry point.
#include "common.cuh"

// Checkpoint scratch shared by all gs_grad_static calls on a device.
static __device__ __align__(256) unsigned char g_static_scratch[GS_STATIC_SCRATCH_BYTES];

namespace {

// The device address of g_static_scratch in the current device's context.  In
// host code the array's name is only a host-side stand-in, so the address is
// looked up with the device current.  It is looked up on every call, not kept:
// a context torn down and created again (cudaDeviceReset) loads the module
// anew, possibly at another address, and a kept pointer would then be stale.
// After the first call on a device the lookup costs no device work.
gs_status scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return GS_ECUDA;
  *out = p;
  return GS_OK;
}

}  // namespace

extern "C" GS_API gs_status gs_grad_static(const gs_problem* prob, const gs_mesh* mesh, const gs_loss* loss_desc,
                                           void* loss, void* dp, void* du0, void* dshared, void* stream) {
  if (!prob || !mesh) return GS_EINVAL;
  if (prob->n == 0) return gs_grad(prob, mesh, loss_desc, loss, dp, du0, dshared, nullptr, 0, stream);
  const size_t need = gs_workspace_bytes(prob, mesh, GS_OP_GRAD);
  if (need == 0) return gs_grad(prob, mesh, loss_desc, loss, dp, du0, dshared, nullptr, 0, stream);
  if (need > (size_t)GS_STATIC_SCRATCH_BYTES) return GS_EWORKSPACE;
  void* ws = nullptr;
  gs_status rc = scratch_address(&ws);
  if (rc != GS_OK) return rc;
  return gs_grad(prob, mesh, loss_desc, loss, dp, du0, dshared, ws, (size_t)GS_STATIC_SCRATCH_BYTES, stream);
}
