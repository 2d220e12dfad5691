// CLA depthwise 3x3 convolution (RIB/SST write-up section 2.3,
// G = PWConv(DWConv3x3(X_2d))): one 3x3 filter and bias per channel, zero
// padding 1 at the image border, channels-last bf16 in and out, fp32 math.
//
// HBM-bound stencil (1 load and 1 store per element, 18 flops per element).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rib_internal.h"
#include "sm100.cuh"

namespace rib {

namespace {

// One thread = one output pixel x 4 consecutive channels (an 8-byte vector).
// Consecutive threads take consecutive channel groups, then consecutive
// columns, so each warp load is a contiguous run of a channels-last row; the
// nine neighbourhood loads of a thread are independent (memory-level
// parallelism), and the overlap between neighbouring threads is served by
// L1/L2, so HBM sees each input byte about once.
__global__ void __launch_bounds__(256) dwconv3x3_kernel(const __nv_bfloat16* __restrict__ X,
                                                        const float* __restrict__ Wdw,
                                                        const float* __restrict__ bdw,
                                                        __nv_bfloat16* __restrict__ out, int B, int H, int W,
                                                        int C) {
  const int cg = C / 4;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long total = static_cast<long long>(B) * H * W * cg;
  if (gid >= total) return;
  const int g = static_cast<int>(gid % cg);
  const long long pix = gid / cg;
  const int x = static_cast<int>(pix % W);
  const int y = static_cast<int>((pix / W) % H);
  const int c = g * 4;
  const size_t rs = static_cast<size_t>(W) * C;
  const __nv_bfloat16* center = X + static_cast<size_t>(pix) * C + c;

  uint2 v[9];
#pragma unroll
  for (int dy = -1; dy <= 1; ++dy) {
#pragma unroll
    for (int dx = -1; dx <= 1; ++dx) {
      const bool ok = (y + dy >= 0) && (y + dy < H) && (x + dx >= 0) && (x + dx < W);
      const __nv_bfloat16* p = center + static_cast<ptrdiff_t>(dy) * static_cast<ptrdiff_t>(rs) + dx * C;
      v[(dy + 1) * 3 + dx + 1] = ok ? __ldg(reinterpret_cast<const uint2*>(p)) : make_uint2(0u, 0u);
    }
  }
  float acc[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] = __ldg(bdw + c + e);
#pragma unroll
  for (int k = 0; k < 9; ++k) {
    const float4 w = make_float4(__ldg(Wdw + (c + 0) * 9 + k), __ldg(Wdw + (c + 1) * 9 + k),
                                 __ldg(Wdw + (c + 2) * 9 + k), __ldg(Wdw + (c + 3) * 9 + k));
    acc[0] = fmaf(w.x, bf16_lo(v[k].x), acc[0]);
    acc[1] = fmaf(w.y, bf16_hi(v[k].x), acc[1]);
    acc[2] = fmaf(w.z, bf16_lo(v[k].y), acc[2]);
    acc[3] = fmaf(w.w, bf16_hi(v[k].y), acc[3]);
  }
  *reinterpret_cast<uint2*>(out + static_cast<size_t>(pix) * C + c) =
      make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
}

}  // namespace

cudaError_t launch_dwconv3x3(const void* X, const float* Wdw, const float* bdw, void* out, int B, int H, int W,
                             int C, cudaStream_t stream) {
  const long long total = static_cast<long long>(B) * H * W * (C / 4);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  dwconv3x3_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(X), Wdw, bdw, static_cast<__nv_bfloat16*>(out), B, H, W, C);
  return cudaGetLastError();
}

}  // namespace rib
