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
#include <mutex>

#include "rib_internal.h"

// The scratch: one per device that loads this library, held until the
// process exits. In host code this name is only a host-side handle for the
// symbol, never a usable device address; the address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char rib_gate_scratch[RIB_GATE_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDev = 64;
void* g_scratch_ptr[kMaxDev] = {nullptr};
std::mutex g_scratch_mu;

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
}  // namespace

using namespace rib;

extern "C" rib_status cla_gate_static_scratch(const void* X, rib_dtype xdtype, int B, int H, int W, int C,
                                              const float* Wdw, const float* bdw, const void* Wpw, const float* bpw,
                                              void* sig_gate, cudaStream_t stream) {
  if (!X || !Wdw || !bdw || !Wpw || !bpw || !sig_gate)
    return fail(RIB_ERR_INVALID_ARG, "cla_gate_static_scratch: null pointer");
  if (B <= 0 || H <= 0 || W <= 0 || C <= 0)
    return fail(RIB_ERR_INVALID_ARG, "cla_gate_static_scratch: sizes must be positive");
  if (C % 4 || C > 256) return fail(RIB_ERR_UNSUPPORTED, "cla_gate_static_scratch: needs C % 4 == 0 and C <= 256");
  if (xdtype == RIB_F32)
    return fail(RIB_ERR_UNSUPPORTED, "cla_gate_static_scratch: convert f32 maps with rib_f32_to_bf16 first");
  const size_t need = static_cast<size_t>(B) * H * W * C * 2;
  if (need > RIB_GATE_STATIC_SCRATCH_BYTES) {
    char buf[200];
    std::snprintf(buf, sizeof(buf),
                  "cla_gate_static_scratch: B*H*W*C*2 = %zu bytes exceeds the fixed scratch of %zu bytes; "
                  "use cla_gate with a workspace",
                  need, static_cast<size_t>(RIB_GATE_STATIC_SCRATCH_BYTES));
    return fail(RIB_ERR_UNSUPPORTED, buf);
  }
  if (!is_aligned(X, 16) || !is_aligned(sig_gate, 16))
    return fail(RIB_ERR_ALIGNMENT, "cla_gate_static_scratch: X and sig_gate need 16-byte alignment");
  if (!is_aligned(Wdw, 4) || !is_aligned(bdw, 4) || !is_aligned(bpw, 4) || !is_aligned(Wpw, 2))
    return fail(RIB_ERR_ALIGNMENT, "cla_gate_static_scratch: fp32 weights 4-byte, Wpw 2-byte aligned");

  // Set-up, once per device, with that device current: the device address
  // of this library's scratch array on it.
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cla_gate_static_scratch: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDev) return fail(RIB_ERR_UNSUPPORTED, "cla_gate_static_scratch: device index out of range");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, rib_gate_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cla_gate_static_scratch: cudaGetSymbolAddress");
      g_scratch_ptr[dev] = ptr;
    }
    scratch = g_scratch_ptr[dev];
  }

  // depthwise 3x3 into the scratch (every element the pointwise step reads is
  // written here first, so nothing needs clearing), then pointwise + sigmoid
  e = launch_dwconv3x3(X, Wdw, bdw, scratch, B, H, W, C, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cla_gate_static_scratch: depthwise launch");
  GemmLaunch g{};
  g.A = scratch;
  g.B = B;
  g.H = H;
  g.W = W;
  g.Hp = H;
  g.Wp = W;
  g.K = C;
  g.mode = 1;
  g.n_real = C;
  g.w_cols = C;
  g.njobs = 1;
  g.jobs[0] = GemmJob{Wpw, sig_gate, (C + 15) / 16 * 16, 0, 0, -1, 1.0f, bpw};
  e = launch_token_gemm(g, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cla_gate_static_scratch: pointwise launch");
  return RIB_OK;
}
