// cla_gate_static_scratch: the CLA gate for callers that cannot allocate
// device memory.
//
// cla_gate needs a caller-provided workspace for its depthwise intermediate.
// Some callers cannot provide one: hosts that forbid device allocation after
// start-up (deployment runtimes with a fixed memory plan, plugin interfaces
// that hand over only inputs and outputs). This entry point keeps that
// intermediate in a fixed array owned by the library instead, so a call
// needs nothing beyond its inputs and outputs and never allocates.
#include <cuda_runtime.h>

#include <cstdio>

#include "rib_internal.h"

// The scratch: one per device that loads this library, held until the
// process exits. In host code this name is only a host-side handle for the
// symbol, never a usable device address; the address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char rib_gate_scratch[RIB_GATE_STATIC_SCRATCH_BYTES];

using namespace rib;

extern "C" rib_status cla_gate_static_scratch(const void* X, rib_dtype xdtype, int B, int H, int W, int C,
                                              const float* Wdw, const float* bdw, const void* Wpw, const float* bpw,
                                              void* sig_gate, cudaStream_t stream) {
  rib_status st = check_gate_args("cla_gate_static_scratch", X, xdtype, B, H, W, C, Wdw, bdw, Wpw, bpw, sig_gate);
  if (st != RIB_OK) return st;
  if (xdtype != RIB_BF16)
    return fail(RIB_ERR_UNSUPPORTED, "cla_gate_static_scratch: X must be bf16 (convert f32 maps with rib_f32_to_bf16)");
  const size_t need = static_cast<size_t>(B) * H * W * C * 2;
  if (need > RIB_GATE_STATIC_SCRATCH_BYTES) {
    char buf[200];
    std::snprintf(buf, sizeof(buf),
                  "cla_gate_static_scratch: B*H*W*C*2 = %zu bytes exceeds the fixed scratch of %zu bytes; "
                  "use cla_gate with a workspace",
                  need, static_cast<size_t>(RIB_GATE_STATIC_SCRATCH_BYTES));
    return fail(RIB_ERR_UNSUPPORTED, buf);
  }
  // Set-up, once per device, with that device current: the device address
  // of this library's scratch array on it (cached by the library).
  cudaError_t e;
  void* scratch = cached_symbol_address(kSymGateScratch, &rib_gate_scratch, &e);
  if (!scratch) return cuda_fail(e == cudaSuccess ? cudaErrorInvalidDevice : e, "cla_gate_static_scratch: cudaGetSymbolAddress");
  // depthwise 3x3 into the scratch (every element the pointwise step reads is
  // written there first, so nothing needs clearing), then pointwise + sigmoid
  return cla_gate_two_pass("cla_gate_static_scratch", X, B, H, W, C, Wdw, bdw, Wpw, bpw, sig_gate, scratch, stream);
}
