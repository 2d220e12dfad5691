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

#ifndef RIB_DW_PIX
#define RIB_DW_PIX 4
#endif
#ifndef RIB_DW_ROWS
#define RIB_DW_ROWS 8
#endif
#ifndef RIB_DW_MINB
#define RIB_DW_MINB 2
#endif
constexpr int kPix = RIB_DW_PIX;     // output pixels per thread along x
constexpr int kRows = RIB_DW_ROWS;   // output rows per thread (sliding 3-row window)
constexpr int kThreadsDW = 256;

// Grid: x = channel groups x strips of kPix columns, y = groups of kRows
// rows, z = image. Thread = 4 consecutive channels (one 8-byte vector) x
// kPix consecutive pixels x kRows consecutive rows: it keeps a sliding
// window of three input rows of kPix + 2 vectors in registers, so each
// input vector is loaded once per thread (about (kPix + 2) / kPix row loads
// per output row instead of three times that) and reused by up to 9
// outputs (4 x 8 pixels per thread, two CTAs per SM: the fastest of the
// shapes measured on B200); filter taps ([9][C]) and
// biases come from shared memory. Consecutive threads take consecutive
// channel groups, so every warp load is a contiguous run of a channels-last
// row.
__device__ __forceinline__ void dw_load_row(const __nv_bfloat16* img, size_t rs, int yy, int H, int x0, int W, int C,
                                            uint2 (&v)[kPix + 2]) {
  const bool vy = yy >= 0 && yy < H;
  const __nv_bfloat16* row = img + static_cast<size_t>(vy ? yy : 0) * rs;
#pragma unroll
  for (int j = 0; j < kPix + 2; ++j) {
    const int xx = x0 + j - 1;
    v[j] = (vy && xx >= 0 && xx < W) ? __ldg(reinterpret_cast<const uint2*>(row + static_cast<size_t>(xx) * C))
                                     : make_uint2(0u, 0u);
  }
}

__global__ void __launch_bounds__(kThreadsDW, RIB_DW_MINB) dwconv3x3_kernel(const __nv_bfloat16* __restrict__ X,
                                                               const float* __restrict__ Wdw,
                                                               const float* __restrict__ bdw,
                                                               __nv_bfloat16* __restrict__ out, int B, int H, int W,
                                                               int C) {
  extern __shared__ float s_w[];      // [9][C] taps (tap-major) then [C] biases
  for (int i = threadIdx.x; i < C * 10; i += blockDim.x) {
    if (i < C * 9) {
      const int t = i / C, c = i - t * C;
      s_w[i] = Wdw[c * 9 + t];
    } else {
      s_w[i] = bdw[i - C * 9];
    }
  }
  __syncthreads();
  const int cg = C / 4;
  const int strips = (W + kPix - 1) / kPix;
  const int gid = blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= strips * cg) return;
  const int g = gid % cg;
  const int x0 = (gid / cg) * kPix;
  const int y0 = blockIdx.y * kRows, b = blockIdx.z;
  const int c = g * 4;
  const size_t rs = static_cast<size_t>(W) * C;
  const __nv_bfloat16* img = X + static_cast<size_t>(b) * H * rs + c;
  const float4 bias = *reinterpret_cast<const float4*>(&s_w[C * 9 + c]);

  uint2 r0[kPix + 2], r1[kPix + 2], r2[kPix + 2];
  dw_load_row(img, rs, y0 - 1, H, x0, W, C, r0);
  dw_load_row(img, rs, y0, H, x0, W, C, r1);
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const int y = y0 + k;
    if (y >= H) break;
    dw_load_row(img, rs, y + 1, H, x0, W, C, r2);
    float acc[kPix][4];
#pragma unroll
    for (int p = 0; p < kPix; ++p) {
      acc[p][0] = bias.x;
      acc[p][1] = bias.y;
      acc[p][2] = bias.z;
      acc[p][3] = bias.w;
    }
#pragma unroll
    for (int dy = 0; dy < 3; ++dy) {
      const uint2* v = dy == 0 ? r0 : (dy == 1 ? r1 : r2);
#pragma unroll
      for (int dx = 0; dx < 3; ++dx) {
        const float4 w = *reinterpret_cast<const float4*>(&s_w[(dy * 3 + dx) * C + c]);
#pragma unroll
        for (int p = 0; p < kPix; ++p) {
          const uint2 u = v[p + dx];
          acc[p][0] = fmaf(w.x, bf16_lo(u.x), acc[p][0]);
          acc[p][1] = fmaf(w.y, bf16_hi(u.x), acc[p][1]);
          acc[p][2] = fmaf(w.z, bf16_lo(u.y), acc[p][2]);
          acc[p][3] = fmaf(w.w, bf16_hi(u.y), acc[p][3]);
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
    // slide the window down one row
#pragma unroll
    for (int j = 0; j < kPix + 2; ++j) {
      r0[j] = r1[j];
      r1[j] = r2[j];
    }
  }
}

}  // namespace

cudaError_t launch_dwconv3x3(const void* X, const float* Wdw, const float* bdw, void* out, int B, int H, int W,
                             int C, cudaStream_t stream) {
  const int per_row = ((W + kPix - 1) / kPix) * (C / 4);
  if (per_row == 0 || H == 0 || B == 0) return cudaSuccess;
  dim3 grid((per_row + kThreadsDW - 1) / kThreadsDW, (H + kRows - 1) / kRows, B);
  dwconv3x3_kernel<<<grid, kThreadsDW, C * 10 * sizeof(float), stream>>>(
      static_cast<const __nv_bfloat16*>(X), Wdw, bdw, static_cast<__nv_bfloat16*>(out), B, H, W, C);
  return cudaGetLastError();
}

}  // namespace rib
