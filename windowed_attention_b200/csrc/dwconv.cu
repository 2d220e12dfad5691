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

constexpr int kPix = 8;        // output pixels per thread along x
constexpr int kThreadsDW = 256;

// Grid: x = channel groups x strips of kPix columns of one row, y = row,
// z = image. Thread = 4 consecutive channels (one 8-byte vector) x kPix
// consecutive pixels: it loads the 3 x (kPix+2) neighbourhood once (rows
// y-1..y+1), keeps it in registers and reuses each vector for up to 3
// outputs; filter taps and biases come from shared memory. Consecutive
// threads take consecutive channel groups, so every warp load is a
// contiguous run of a channels-last row.
__global__ void __launch_bounds__(kThreadsDW) dwconv3x3_kernel(const __nv_bfloat16* __restrict__ X,
                                                               const float* __restrict__ Wdw,
                                                               const float* __restrict__ bdw,
                                                               __nv_bfloat16* __restrict__ out, int B, int H, int W,
                                                               int C) {
  extern __shared__ float s_w[];      // [C][9] taps then [C] biases
  for (int i = threadIdx.x; i < C * 10; i += blockDim.x) s_w[i] = i < C * 9 ? Wdw[i] : bdw[i - C * 9];
  __syncthreads();
  const int cg = C / 4;
  const int strips = (W + kPix - 1) / kPix;
  const int gid = blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= strips * cg) return;
  const int g = gid % cg;
  const int x0 = (gid / cg) * kPix;
  const int y = blockIdx.y, b = blockIdx.z;
  const int c = g * 4;
  const size_t rs = static_cast<size_t>(W) * C;
  const __nv_bfloat16* img = X + static_cast<size_t>(b) * H * rs + c;

  float acc[kPix][4];
#pragma unroll
  for (int p = 0; p < kPix; ++p)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[p][e] = s_w[C * 9 + c + e];
#pragma unroll
  for (int dy = 0; dy < 3; ++dy) {
    const int yy = y + dy - 1;
    const bool vy = yy >= 0 && yy < H;
    const __nv_bfloat16* row = img + static_cast<size_t>(vy ? yy : 0) * rs;
    uint2 v[kPix + 2];
#pragma unroll
    for (int j = 0; j < kPix + 2; ++j) {
      const int xx = x0 + j - 1;
      v[j] = (vy && xx >= 0 && xx < W) ? __ldg(reinterpret_cast<const uint2*>(row + static_cast<size_t>(xx) * C))
                                       : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int dx = 0; dx < 3; ++dx) {
      float w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) w[e] = s_w[(c + e) * 9 + dy * 3 + dx];
#pragma unroll
      for (int p = 0; p < kPix; ++p) {
        const uint2 u = v[p + dx];
        acc[p][0] = fmaf(w[0], bf16_lo(u.x), acc[p][0]);
        acc[p][1] = fmaf(w[1], bf16_hi(u.x), acc[p][1]);
        acc[p][2] = fmaf(w[2], bf16_lo(u.y), acc[p][2]);
        acc[p][3] = fmaf(w[3], bf16_hi(u.y), acc[p][3]);
      }
    }
  }
  __nv_bfloat16* orow = out + (static_cast<size_t>(b) * H + y) * rs + c;
#pragma unroll
  for (int p = 0; p < kPix; ++p) {
    if (x0 + p < W)
      *reinterpret_cast<uint2*>(orow + static_cast<size_t>(x0 + p) * C) =
          make_uint2(pack_bf16x2(acc[p][0], acc[p][1]), pack_bf16x2(acc[p][2], acc[p][3]));
  }
}

}  // namespace

cudaError_t launch_dwconv3x3(const void* X, const float* Wdw, const float* bdw, void* out, int B, int H, int W,
                             int C, cudaStream_t stream) {
  const int per_row = ((W + kPix - 1) / kPix) * (C / 4);
  if (per_row == 0 || H == 0 || B == 0) return cudaSuccess;
  dim3 grid((per_row + kThreadsDW - 1) / kThreadsDW, H, B);
  dwconv3x3_kernel<<<grid, kThreadsDW, C * 10 * sizeof(float), stream>>>(
      static_cast<const __nv_bfloat16*>(X), Wdw, bdw, static_cast<__nv_bfloat16*>(out), B, H, W, C);
  return cudaGetLastError();
}

}  // namespace rib
