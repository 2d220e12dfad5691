// Backward of the layer's two token-wise parts: the content projections and
// the CLA gate (RIB/SST write-up section 2.3; the projections are the
// content features of "Résumé technique" 2.A). With g_j the gradients of the
// projection outputs (j = q, k, v; Qc carries q_scale) and dG the gradient of
// the gate pre-activation G = D Wpw + bpw, D = DWConv3x3(X):
//   dX   = sum_j (s_j g_j) W_j^T  +  DWConv3x3^T(dD),   dD = dG Wpw^T
//   dW_j = X^T (s_j g_j),  dWpw = D^T dG,  dbpw = sum_t dG,
//   dWdw[c][ky][kx] = sum_p X[p + (ky-1, kx-1)][c] dD[p][c],  dbdw = sum_t dD.
// The token GEMMs (dX, dD) and the weight-gradient reductions (dW_j, dWpw) run
// on tcgen05 (layer_bwd_tc.cu) for maps whose rows the bulk copies can move
// (W*C % 8 == 0, 16-byte aligned); the fp32 CUDA-core tiled kernels below
// take the other maps. Every reduction over tokens writes partial sums that a
// second kernel adds in a fixed order (no atomics), so all gradients are
// bit-identical from run to run. The depthwise parts are elementwise /
// reduction kernels.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rib_internal.h"
#include "sm100.cuh"

namespace rib {

namespace {

constexpr int kBM = 64, kBN = 64, kBK = 32, kThr = 256;

__device__ __forceinline__ float bf2f(__nv_bfloat16 v) { return __bfloat162float(v); }

// Token GEMM out[t][n] = sum_kk A(t, kk) * Bw(kk, n), fp32 accumulate.
//  MODE 0 (projection input gradient): kk = j*C + h*dh + d over the three
//    jobs; A(t, kk) = s_j * g_j[tp(t)][h][d] with g_j fp32 in the padded
//    layout [B][Hp][Wp][heads][32] and tp the padded token of image token t;
//    Bw(kk, n) = W_j[n][h*dh + d] (bf16 [C][C], out = dX fp32 [T][C]).
//  MODE 1 (gate): kk over C; A(t, kk) = dG[t][kk] (bf16 [T][C]);
//    Bw(kk, n) = Wpw[n][kk]; out = dD fp32 [T][C].
struct TokGemm {
  int B, H, W, Hp, Wp, C, heads, dh;
  long long T;
  const float* g[3];
  float s[3];
  const __nv_bfloat16* Wt[3];
  const __nv_bfloat16* dG;
  float* out;
};

constexpr int kMaxKK = 3 * 256;

template <int MODE>
__global__ void __launch_bounds__(kThr) tok_gemm_kernel(const TokGemm p) {
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs[kBK][kBN + 4];
  __shared__ long long s_base[kBM];   // MODE 0: padded token * heads * 32 (-1 past T)
  // per reduction index kk: job j, offset of (h, d) inside a padded g row,
  // and weight column r = h*dh + d (MODE 0); tables replace per-element
  // integer divisions in the tile loads
  __shared__ short s_kj[kMaxKK], s_koff[kMaxKK], s_kr[kMaxKK];
  const int tid = threadIdx.x;
  const long long t0 = static_cast<long long>(blockIdx.x) * kBM;
  const int n0 = blockIdx.y * kBN;
  const int C = p.C;
  const int KK = MODE == 0 ? 3 * C : C;
  for (int kk = tid; kk < KK; kk += kThr) {
    const int j = MODE == 0 ? kk / C : 0;
    const int r = kk - j * C;
    s_kj[kk] = static_cast<short>(j);
    s_kr[kk] = static_cast<short>(r);
    s_koff[kk] = static_cast<short>(MODE == 0 ? (r / p.dh) * 32 + r % p.dh : r);
  }
  if (tid < kBM) {
    const long long t = t0 + tid;
    long long base = -1;
    if (t < p.T) {
      if (MODE == 0) {
        const long long hw = static_cast<long long>(p.H) * p.W;
        const int b = static_cast<int>(t / hw);
        const int rem = static_cast<int>(t - b * hw);
        const int y = rem / p.W, x = rem - (rem / p.W) * p.W;
        base = ((static_cast<long long>(b) * p.Hp + y) * p.Wp + x) * p.heads * 32;
      } else {
        base = t * C;
      }
    }
    s_base[tid] = base;
  }
  __syncthreads();
  const int tm = tid / 16, tn = tid % 16;   // 4x4 outputs: rows 4tm.., cols 4tn..
  float acc[4][4] = {};
  for (int k0 = 0; k0 < KK; k0 += kBK) {
    // A tile: thread loads column kc of rows r, r + 8, ...
    {
      const int kc = tid % kBK, kk = k0 + kc;
      int off = -1, j = 0;
      float sc = 1.f;
      if (kk < KK) {
        off = s_koff[kk];
        if (MODE == 0) {
          j = s_kj[kk];
          sc = j == 0 ? p.s[0] : (j == 1 ? p.s[1] : p.s[2]);
        }
      }
      const float* gj = MODE == 0 ? (j == 0 ? p.g[0] : (j == 1 ? p.g[1] : p.g[2])) : nullptr;
      for (int m = tid / kBK; m < kBM; m += kThr / kBK) {
        const long long base = s_base[m];
        float v = 0.f;
        if (off >= 0 && base >= 0) v = MODE == 0 ? gj[base + off] * sc : bf2f(p.dG[base + off]);
        As[kc][m] = v;
      }
    }
    // B tile: thread loads 8 consecutive kk of output column n
    {
      const int nl = tid / 4, n = n0 + nl;
      for (int e = 0; e < 8; ++e) {
        const int kc = 8 * (tid % 4) + e, kk = k0 + kc;
        float v = 0.f;
        if (kk < KK && n < C) {
          if (MODE == 0) {
            const int j = s_kj[kk], r = s_kr[kk];
            const __nv_bfloat16* Wj = j == 0 ? p.Wt[0] : (j == 1 ? p.Wt[1] : p.Wt[2]);
            v = bf2f(Wj[static_cast<size_t>(n) * C + r]);
          } else {
            v = bf2f(p.Wt[0][static_cast<size_t>(n) * C + kk]);
          }
        }
        Bs[kc][nl] = v;
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int kc = 0; kc < kBK; ++kc) {
      const float4 a = *reinterpret_cast<const float4*>(&As[kc][4 * tm]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[kc][4 * tn]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(av[i], bv[q], acc[i][q]);
    }
    __syncthreads();
  }
  for (int i = 0; i < 4; ++i) {
    const long long t = t0 + 4 * tm + i;
    if (t >= p.T) break;
    for (int q = 0; q < 4; ++q) {
      const int n = n0 + 4 * tn + q;
      if (n < C) p.out[t * C + n] = acc[i][q];
    }
  }
}

// Weight gradient dW[c][n] = sum_t Xa(t, c) * G(t, n) over a chunk of tokens
// per block, written to partial[chunk][job][c][n] (chunk = blockIdx.y, job =
// blockIdx.z); the chunks are added in order afterwards.
//  MODE 0: Xa = X (bf16 [T][C]); G(t, n) = s_j g_j[tp(t)][h][d], n = h*dh + d;
//          blockIdx.z = job j, dW = dW_j.
//  MODE 1: Xa = D (bf16 [T][C]); G = dG (bf16 [T][C]); dW = dWpw.
struct WGrad {
  int B, H, W, Hp, Wp, C, heads, dh, tchunk;
  long long T;
  const __nv_bfloat16* Xa;
  const float* g[3];
  float s[3];
  const __nv_bfloat16* dG;
  float* partial;
};

template <int MODE>
__global__ void __launch_bounds__(kThr) wgrad_kernel(const WGrad p) {
  __shared__ float Xs[kBK][kBM + 4];
  __shared__ float Gs[kBK][kBN + 4];
  __shared__ long long s_gbase[kBK];   // MODE 0: padded token * heads * 32 of the chunk's rows
  const int tid = threadIdx.x;
  const int C = p.C;
  const int m0 = (blockIdx.x % ((C + kBM - 1) / kBM)) * kBM;
  const int n0 = (blockIdx.x / ((C + kBM - 1) / kBM)) * kBN;
  const int j = MODE == 0 ? blockIdx.z : 0;
  const float* gj = j == 0 ? p.g[0] : (j == 1 ? p.g[1] : p.g[2]);
  const float sj = j == 0 ? p.s[0] : (j == 1 ? p.s[1] : p.s[2]);
  float* dW = p.partial + (static_cast<size_t>(blockIdx.y) * gridDim.z + j) * p.C * p.C;
  const long long tb = static_cast<long long>(blockIdx.y) * p.tchunk;
  const long long te = tb + p.tchunk < p.T ? tb + p.tchunk : p.T;
  const int tm = tid / 16, tn = tid % 16;
  float acc[4][4] = {};
  // G column offset of this thread's loads (MODE 0: head-padded position)
  const int lc = tid % 64;
  const int n_ld = n0 + lc;
  const int goff = MODE == 0 ? (n_ld < C ? (n_ld / p.dh) * 32 + n_ld % p.dh : -1) : (n_ld < C ? n_ld : -1);
  const int c_ld = m0 + lc;
  for (long long k0 = tb; k0 < te; k0 += kBK) {
    if (MODE == 0 && tid < kBK) {
      const long long t = k0 + tid;
      long long base = 0;
      if (t < te) {
        const long long hw = static_cast<long long>(p.H) * p.W;
        const int b = static_cast<int>(t / hw);
        const int rem = static_cast<int>(t - b * hw);
        const int y = rem / p.W, x = rem - (rem / p.W) * p.W;
        base = ((static_cast<long long>(b) * p.Hp + y) * p.Wp + x) * p.heads * 32;
      }
      s_gbase[tid] = base;
    }
    if (MODE == 0) __syncthreads();
    for (int r = tid / 64; r < kBK; r += kThr / 64) {
      const long long t = k0 + r;
      float xv = 0.f, gv = 0.f;
      if (t < te) {
        if (c_ld < C) xv = bf2f(p.Xa[t * C + c_ld]);
        if (goff >= 0) {
          if (MODE == 0) {
            gv = gj[s_gbase[r] + goff] * sj;
          } else {
            gv = bf2f(p.dG[t * C + goff]);
          }
        }
      }
      Xs[r][lc] = xv;
      Gs[r][lc] = gv;
    }
    __syncthreads();
#pragma unroll 8
    for (int kc = 0; kc < kBK; ++kc) {
      const float4 a = *reinterpret_cast<const float4*>(&Xs[kc][4 * tm]);
      const float4 b = *reinterpret_cast<const float4*>(&Gs[kc][4 * tn]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(av[i], bv[q], acc[i][q]);
    }
    __syncthreads();
  }
  for (int i = 0; i < 4; ++i) {
    const int c = m0 + 4 * tm + i;
    if (c >= C) break;
    for (int q = 0; q < 4; ++q) {
      const int n = n0 + 4 * tn + q;
      if (n < C) dW[static_cast<size_t>(c) * C + n] = acc[i][q];
    }
  }
}

// dX[b,y,x,c] += sum_{ky,kx} Wdw[c][ky][kx] * dD[b, y+1-ky, x+1-kx, c]
// (the transposed depthwise conv, zero outside the image). Thread = 4
// channels x a run of kDxRun pixels of one row: the taps are loaded once per
// run and each input row's kDxRun + 2 values serve all of the run's outputs.
constexpr int kDxRun = 8;
__global__ void __launch_bounds__(kThr) dw_dx_kernel(const float* __restrict__ dD, const float* __restrict__ Wdw,
                                                     float* __restrict__ dX, int B, int H, int W, int C) {
  const int cq = C / 4;
  const int nrun = (W + kDxRun - 1) / kDxRun;
  const long long i = static_cast<long long>(blockIdx.x) * kThr + threadIdx.x;
  const long long n = static_cast<long long>(B) * H * nrun * cq;
  if (i >= n) return;
  const int q = static_cast<int>(i % cq);
  const long long rest = i / cq;
  const int x0 = static_cast<int>(rest % nrun) * kDxRun;
  const long long row = rest / nrun;   // b * H + y
  const int y = static_cast<int>(row % H);
  const long long b = row / H;
  float w[4][9];
#pragma unroll
  for (int e = 0; e < 4; ++e)
#pragma unroll
    for (int t = 0; t < 9; ++t) w[e][t] = __ldg(Wdw + (4 * q + e) * 9 + t);
  float4 acc[kDxRun];
#pragma unroll
  for (int k = 0; k < kDxRun; ++k)
    acc[k] = (x0 + k < W) ? reinterpret_cast<const float4*>(dX)[((row * W) + x0 + k) * cq + q] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int ky = 0; ky < 3; ++ky) {
    const int ys = y + 1 - ky;
    if (ys < 0 || ys >= H) continue;
    // dD at columns x0-1 .. x0+kDxRun of row ys (zero outside the image)
    float4 d[kDxRun + 2];
#pragma unroll
    for (int k = 0; k < kDxRun + 2; ++k) {
      const int xs = x0 - 1 + k;
      d[k] = (xs >= 0 && xs < W) ? __ldg(reinterpret_cast<const float4*>(dD) + ((b * H + ys) * W + xs) * cq + q)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < kDxRun; ++k) {
#pragma unroll
      for (int kx = 0; kx < 3; ++kx) {
        const float4 v = d[k + 2 - kx];   // column x0 + k + 1 - kx
        const int t = ky * 3 + kx;
        acc[k].x = fmaf(w[0][t], v.x, acc[k].x);
        acc[k].y = fmaf(w[1][t], v.y, acc[k].y);
        acc[k].z = fmaf(w[2][t], v.z, acc[k].z);
        acc[k].w = fmaf(w[3][t], v.w, acc[k].w);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < kDxRun; ++k)
    if (x0 + k < W) reinterpret_cast<float4*>(dX)[((row * W) + x0 + k) * cq + q] = acc[k];
}

// Per-channel reductions over all pixels: dWdw[c][ky][kx] = sum X[p + (ky-1,
// kx-1)][c] dD[p][c], dbdw[c] = sum dD[p][c], dbpw[c] = sum dG[p][c].
// One block per rpb consecutive map rows; threadIdx.x = channel quad,
// threadIdx.y = a lane over the rows' runs of kDxRun pixels (each input row's
// kDxRun + 2 values serve the whole run); the block's sums (reduced in shared
// memory in a fixed order) go to part[block][c][11]; dw_final_kernel adds the
// blocks in order.
constexpr int kRedY = 8;
__global__ void dw_reduce_kernel(const __nv_bfloat16* __restrict__ X, const float* __restrict__ dD,
                                 const __nv_bfloat16* __restrict__ dG, float* __restrict__ part, int B, int H, int W,
                                 int C, int rpb) {
  extern __shared__ float red[];   // [kRedY][C/4][4][11]
  const int cq = C / 4;
  const int q = threadIdx.x, ly = threadIdx.y;
  const long long rows = static_cast<long long>(B) * H;
  const long long r0 = static_cast<long long>(blockIdx.x) * rpb;
  const int nrow = rows - r0 < rpb ? static_cast<int>(rows - r0) : rpb;
  const int nrun = (W + kDxRun - 1) / kDxRun;
  float acc[4][11] = {};
  if (q < cq) {
    for (int jr = ly; jr < nrow * nrun; jr += kRedY) {
      const long long row = r0 + jr / nrun;   // b * H + y
      const int y = static_cast<int>(row % H);
      const long long b = row / H;
      const int x0 = (jr % nrun) * kDxRun;
      float4 d[kDxRun];
#pragma unroll
      for (int k = 0; k < kDxRun; ++k) {
        const int x = x0 + k;
        d[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (x < W) {
          const long long pix = row * W + x;
          d[k] = __ldg(reinterpret_cast<const float4*>(dD) + pix * cq + q);
          const uint2 gw = __ldg(reinterpret_cast<const uint2*>(dG) + pix * cq + q);
          acc[0][9] += d[k].x;
          acc[1][9] += d[k].y;
          acc[2][9] += d[k].z;
          acc[3][9] += d[k].w;
          acc[0][10] += bf16_lo(gw.x);
          acc[1][10] += bf16_hi(gw.x);
          acc[2][10] += bf16_lo(gw.y);
          acc[3][10] += bf16_hi(gw.y);
        }
      }
#pragma unroll
      for (int ky = 0; ky < 3; ++ky) {
        const int ys = y + ky - 1;
        if (ys < 0 || ys >= H) continue;
        // X at columns x0-1 .. x0+kDxRun of row ys (zero outside the image)
        uint2 xw[kDxRun + 2];
#pragma unroll
        for (int k = 0; k < kDxRun + 2; ++k) {
          const int xs = x0 - 1 + k;
          xw[k] = (xs >= 0 && xs < W) ? __ldg(reinterpret_cast<const uint2*>(X) + ((b * H + ys) * W + xs) * cq + q)
                                      : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < kDxRun; ++k) {
#pragma unroll
          for (int kx = 0; kx < 3; ++kx) {
            const uint2 v = xw[k + kx];   // column x0 + k + kx - 1
            const int t = ky * 3 + kx;
            acc[0][t] = fmaf(bf16_lo(v.x), d[k].x, acc[0][t]);
            acc[1][t] = fmaf(bf16_hi(v.x), d[k].y, acc[1][t]);
            acc[2][t] = fmaf(bf16_lo(v.y), d[k].z, acc[2][t]);
            acc[3][t] = fmaf(bf16_hi(v.y), d[k].w, acc[3][t]);
          }
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int v = 0; v < 11; ++v) red[((ly * cq + q) * 4 + e) * 11 + v] = acc[e][v];
  }
  __syncthreads();
  if (ly == 0 && q < cq) {
    float* out = part + static_cast<size_t>(blockIdx.x) * C * 11;
    for (int e = 0; e < 4; ++e) {
      const int c = 4 * q + e;
      for (int v = 0; v < 11; ++v) {
        float sum = 0.f;
        for (int l = 0; l < kRedY; ++l) sum += red[((l * cq + q) * 4 + e) * 11 + v];
        out[c * 11 + v] = sum;
      }
    }
  }
}

// dWdw, dbdw, dbpw from the blocks' partial sums, added in block order.
__global__ void dw_final_kernel(const float* __restrict__ part, int blocks, int C, float* __restrict__ dWdw,
                                float* __restrict__ dbdw, float* __restrict__ dbpw) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;   // c * 11 + v
  if (i >= C * 11) return;
  float s = 0.f;
  for (int k = 0; k < blocks; ++k) s += part[static_cast<size_t>(k) * C * 11 + i];
  const int c = i / 11, v = i - c * 11;
  if (v < 9) dWdw[c * 9 + v] = s;
  else if (v == 9) dbdw[c] = s;
  else dbpw[c] = s;
}

// rows per block of the depthwise reductions (about two blocks per SM on a
// B200-sized grid of rows) and the number of blocks
int red_rows_per_block(int B, int H) {
  const long long rows = static_cast<long long>(B) * H;
  const long long r = (rows + 295) / 296;
  return static_cast<int>(r < 1 ? 1 : r);
}
long long red_blocks(int B, int H) {
  const long long rows = static_cast<long long>(B) * H;
  const int rpb = red_rows_per_block(B, H);
  return (rows + rpb - 1) / rpb;
}

}  // namespace

size_t qkv_project_bwd_ws_bytes(int B, int H, int W, int C, int heads) {
  (void)B;
  (void)H;
  (void)W;
  return align256(tc_bwd_weight_image_bytes(C, heads, true)) + wgrad_partial_bytes(C);
}

cudaError_t launch_qkv_project_bwd(const QkvBwdLaunch& a, void* ws, cudaStream_t stream) {
  const long long T = static_cast<long long>(a.B) * a.H * a.W;
  if (T == 0) return cudaSuccess;
  if (tc_bwd_supported(a.X, a.H, a.W, a.C)) return launch_qkv_project_bwd_tc(a, ws, stream);
  TokGemm t{};
  t.B = a.B; t.H = a.H; t.W = a.W; t.Hp = a.Hp; t.Wp = a.Wp; t.C = a.C; t.heads = a.heads; t.dh = a.C / a.heads;
  t.T = T;
  for (int j = 0; j < 3; ++j) {
    t.g[j] = a.g[j];
    t.s[j] = a.s[j];
    t.Wt[j] = static_cast<const __nv_bfloat16*>(a.Wt[j]);
  }
  t.out = a.dX;
  dim3 grid(static_cast<unsigned>((T + kBM - 1) / kBM), (a.C + kBN - 1) / kBN);
  tok_gemm_kernel<0><<<grid, kThr, 0, stream>>>(t);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  WGrad w{};
  w.B = a.B; w.H = a.H; w.W = a.W; w.Hp = a.Hp; w.Wp = a.Wp; w.C = a.C; w.heads = a.heads; w.dh = a.C / a.heads;
  w.T = T;
  w.Xa = static_cast<const __nv_bfloat16*>(a.X);
  for (int j = 0; j < 3; ++j) {
    w.g[j] = a.g[j];
    w.s[j] = a.s[j];
  }
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                            align256(tc_bwd_weight_image_bytes(a.C, a.heads, true)));
  w.partial = partial;
  // token chunk per block: about 4 blocks per SM over the 3 x tiles^2 grid,
  // at most kWgradChunks / 3 chunks (the partial buffer's size)
  const int tiles = (a.C + kBM - 1) / kBM;
  long long chunks = 4LL * sm_count() / (3LL * tiles * tiles);
  if (chunks > kWgradChunks / 3) chunks = kWgradChunks / 3;
  if (chunks < 1) chunks = 1;
  long long tchunk = (T + chunks - 1) / chunks;
  tchunk = (tchunk + kBK - 1) / kBK * kBK;
  w.tchunk = static_cast<int>(tchunk);
  const int nchunks = static_cast<int>((T + tchunk - 1) / tchunk);
  dim3 wg(tiles * tiles, nchunks, 3);
  wgrad_kernel<0><<<wg, kThr, 0, stream>>>(w);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_wgrad_partial_sum(partial, nchunks, 3, a.C * a.C, a.dW[0], a.dW[1], a.dW[2], stream);
}

// workspace: dD fp32 [T][C] | weight atoms | partials of dWpw | per-block
// partials of the depthwise reductions
size_t gate_bwd_ws_bytes(int B, int H, int W, int C) {
  const long long T = static_cast<long long>(B) * H * W;
  return align256(static_cast<size_t>(T) * C * 4) + align256(tc_bwd_weight_image_bytes(C, 1, false)) +
         align256(wgrad_partial_bytes(C)) + static_cast<size_t>(red_blocks(B, H)) * C * 11 * 4;
}

cudaError_t launch_cla_gate_bwd(const GateBwdLaunch& a, void* ws, cudaStream_t stream) {
  const long long T = static_cast<long long>(a.B) * a.H * a.W;
  if (T == 0) return cudaSuccess;
  const int C = a.C;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* img = base + align256(static_cast<size_t>(T) * C * 4);
  float* partial = reinterpret_cast<float*>(img + align256(tc_bwd_weight_image_bytes(C, 1, false)));
  float* part2 = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(partial) + align256(wgrad_partial_bytes(C)));
  int chunks = 0;
  cudaError_t e;
  if (tc_bwd_supported(a.dG, a.H, a.W, C) && tc_bwd_supported(a.D, a.H, a.W, C)) {
    // dD = dG Wpw^T and the partials of dWpw = D^T dG on tcgen05
    e = launch_gate_bwd_tc_gemms(a, img, partial, stream, &chunks);
    if (e != cudaSuccess) return e;
  } else {
    // dD = dG Wpw^T
    TokGemm t{};
    t.B = a.B; t.H = a.H; t.W = a.W; t.Hp = a.H; t.Wp = a.W; t.C = C; t.heads = 1; t.dh = C;
    t.T = T;
    t.Wt[0] = static_cast<const __nv_bfloat16*>(a.Wpw);
    t.dG = static_cast<const __nv_bfloat16*>(a.dG);
    t.out = a.dD;
    dim3 grid(static_cast<unsigned>((T + kBM - 1) / kBM), (C + kBN - 1) / kBN);
    tok_gemm_kernel<1><<<grid, kThr, 0, stream>>>(t);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    WGrad w{};
    w.B = a.B; w.H = a.H; w.W = a.W; w.Hp = a.H; w.Wp = a.W; w.C = C; w.heads = 1; w.dh = C;
    w.T = T;
    w.Xa = static_cast<const __nv_bfloat16*>(a.D);
    w.dG = static_cast<const __nv_bfloat16*>(a.dG);
    w.s[0] = 1.f;
    w.partial = partial;
    const int tiles = (C + kBM - 1) / kBM;
    long long nch = 4LL * sm_count() / (tiles * tiles);
    if (nch > kWgradChunks) nch = kWgradChunks;
    if (nch < 1) nch = 1;
    long long tchunk = (T + nch - 1) / nch;
    tchunk = (tchunk + kBK - 1) / kBK * kBK;
    w.tchunk = static_cast<int>(tchunk);
    chunks = static_cast<int>((T + tchunk - 1) / tchunk);
    dim3 wg(tiles * tiles, chunks, 1);
    wgrad_kernel<1><<<wg, kThr, 0, stream>>>(w);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // dX += DWConv3x3^T(dD)
  const long long n4 = static_cast<long long>(a.B) * a.H * ((a.W + kDxRun - 1) / kDxRun) * (C / 4);
  dw_dx_kernel<<<static_cast<unsigned>((n4 + kThr - 1) / kThr), kThr, 0, stream>>>(a.dD, a.Wdw, a.dX, a.B, a.H, a.W, C);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_wgrad_partial_sum(partial, chunks, 1, C * C, a.dWpw, nullptr, nullptr, stream);
  if (e != cudaSuccess) return e;
  // depthwise weight and bias gradients, dbpw
  const int cq = C / 4;
  const size_t shm = static_cast<size_t>(kRedY) * cq * 4 * 11 * sizeof(float);
  if (shm > 48 * 1024) {
    e = cudaFuncSetAttribute(dw_reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(shm));
    if (e != cudaSuccess) return e;
  }
  const long long blocks = red_blocks(a.B, a.H);
  dim3 rb(cq, kRedY);
  dw_reduce_kernel<<<static_cast<unsigned>(blocks), rb, shm, stream>>>(
      static_cast<const __nv_bfloat16*>(a.X), a.dD, static_cast<const __nv_bfloat16*>(a.dG), part2, a.B, a.H, a.W, C,
      red_rows_per_block(a.B, a.H));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dw_final_kernel<<<(C * 11 + 255) / 256, 256, 0, stream>>>(part2, static_cast<int>(blocks), C, a.dWdw, a.dbdw, a.dbpw);
  return cudaGetLastError();
}

}  // namespace rib
