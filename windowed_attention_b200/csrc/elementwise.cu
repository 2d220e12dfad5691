// Small HBM-bound kernels of the path:
//  * LayerNorm over channels per token (RIB/SST write-up section 3.1: each
//    block runs LayerNorm -> RIB attention -> CLA); fp32 statistics, bf16 out;
//  * fp32 -> bf16 rounding of feature maps handed over in fp32;
//  * the position encoder + coordinate MLP (section 2.2), run once per window
//    size and cached (section 5.2).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rib_internal.h"
#include "sm100.cuh"

namespace rib {

namespace {

// One warp per token. Lane l handles the 4-channel groups l, l+32, ...
// XT: 0 bf16, 1 fp32, 2 fp16 input; YF16: fp16 output (else bf16).
template <int XT, bool YF16>
__global__ void __launch_bounds__(256) layernorm_kernel(const void* __restrict__ xin, uint16_t* __restrict__ y,
                                                        long long T, int C, const float* __restrict__ gamma,
                                                        const float* __restrict__ beta, float eps) {
  const long long tok = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (tok >= T) return;
  constexpr int kMaxG = 8;   // C <= 1024
  const int groups = C / 4;
  float v[kMaxG][4];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxG; ++i) {
    const int g = lane + 32 * i;
    if (g < groups) {
      if (XT == 1) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(xin) + tok * C) + g);
        v[i][0] = f.x; v[i][1] = f.y; v[i][2] = f.z; v[i][3] = f.w;
      } else {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(xin) + tok * C) + g);
        if (XT == 2) {
          v[i][0] = f16_lo(u.x); v[i][1] = f16_hi(u.x); v[i][2] = f16_lo(u.y); v[i][3] = f16_hi(u.y);
        } else {
          v[i][0] = bf16_lo(u.x); v[i][1] = bf16_hi(u.x); v[i][2] = bf16_lo(u.y); v[i][3] = bf16_hi(u.y);
        }
      }
      s += (v[i][0] + v[i][1]) + (v[i][2] + v[i][3]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / C;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxG; ++i) {
    const int g = lane + 32 * i;
    if (g < groups) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float d = v[i][e] - mean;
        q = fmaf(d, d, q);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q / C + eps);
#pragma unroll
  for (int i = 0; i < kMaxG; ++i) {
    const int g = lane + 32 * i;
    if (g < groups) {
      float r[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 4 * g + e;
        r[e] = (v[i][e] - mean) * rstd;
        if (gamma) r[e] *= __ldg(gamma + c);
        if (beta) r[e] += __ldg(beta + c);
      }
      reinterpret_cast<uint2*>(y + tok * C)[g] =
          YF16 ? make_uint2(pack_f16x2_sat(r[0], r[1]), pack_f16x2_sat(r[2], r[3]))
               : make_uint2(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]));
    }
  }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y, size_t n) {
  const size_t i = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i + 3 < n) {
    const float4 f = *reinterpret_cast<const float4*>(x + i);
    reinterpret_cast<uint2*>(y + i)[0] = make_uint2(pack_bf16x2(f.x, f.y), pack_bf16x2(f.z, f.w));
  } else {
    for (size_t j = i; j < n; ++j) y[j] = __float2bfloat16_rn(x[j]);
  }
}

__global__ void bf16_to_f32_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ y, size_t n) {
  const size_t i = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i + 3 < n) {
    const uint2 v = *reinterpret_cast<const uint2*>(x + i);
    *reinterpret_cast<float4*>(y + i) = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
  } else {
    for (size_t j = i; j < n; ++j) y[j] = __bfloat162float(x[j]);
  }
}

// Fourier feature e of window token (i, j) (write-up section 2.2
// CoordinateEncoder): the coordinates y_i, x_j on linspace(-1, 1, M), then per
// band b sin(2^b y), sin(2^b x), cos(2^b y), cos(2^b x). The arguments reach
// 2^(L-1) rad, where a float argument alone carries an error up to its ulp
// (2^-9 rad at 2^14), so the coordinates, the 2^b multiples and sin/cos are
// evaluated in double (once per window size: the cost does not matter).
__device__ __forceinline__ float fourier_feature(int M, int i, int j, int e) {
  const double cy = M > 1 ? -1.0 + 2.0 * i / (M - 1) : 0.0;
  const double cx = M > 1 ? -1.0 + 2.0 * j / (M - 1) : 0.0;
  if (e < 2) return static_cast<float>(e == 0 ? cy : cx);
  const int b = (e - 2) >> 2, w = (e - 2) & 3;
  const double a = ldexp(w & 1 ? cx : cy, b);
  return static_cast<float>(w < 2 ? sin(a) : cos(a));
}

// One CTA per window token t = i*M + j: r = Fourier features of (y_i, x_j),
// h = ReLU(r Wh + bh) (threads over the hidden width), then the heads*R
// outputs of Qp = h Wpq (scaled by 1/sqrt(R)) and Kp = h Wpk.
__global__ void __launch_bounds__(256) pos_encode_kernel(int M, int L, int hidden, int heads, int R,
                                                         const float* __restrict__ Wh, const float* __restrict__ bh,
                                                         const float* __restrict__ Wpq, const float* __restrict__ Wpk,
                                                         __nv_bfloat16* __restrict__ qp, __nv_bfloat16* __restrict__ kp,
                                                         float q_scale) {
  __shared__ float r[2 + 4 * 16];
  __shared__ float h[256];
  const int t = blockIdx.x;
  const int i = t / M, j = t % M;
  const int E = 2 + 4 * L;
  if (threadIdx.x < E) r[threadIdx.x] = fourier_feature(M, i, j, threadIdx.x);   // one thread per feature
  __syncthreads();
  for (int k = threadIdx.x; k < hidden; k += blockDim.x) {
    float a = __ldg(bh + k);
    for (int e = 0; e < E; ++e) a = fmaf(r[e], __ldg(Wh + e * hidden + k), a);
    h[k] = fmaxf(a, 0.f);
  }
  __syncthreads();
  const int outs = heads * R;
  const int N = M * M;
  for (int o = threadIdx.x; o < 2 * outs; o += blockDim.x) {
    const bool isq = o < outs;
    const int c = isq ? o : o - outs;
    const float* Wp = isq ? Wpq : Wpk;
    float a = 0.f;
    for (int k = 0; k < hidden; ++k) a = fmaf(h[k], __ldg(Wp + k * outs + c), a);
    const int hd = c / R, rr = c % R;
    const size_t dst = (static_cast<size_t>(hd) * N + t) * R + rr;
    if (isq) qp[dst] = __float2bfloat16_rn(a * q_scale);
    else kp[dst] = __float2bfloat16_rn(a);
  }
}

// Coordinate-MLP backward, step 1, one CTA per window token t: recompute the
// Fourier features r and h = ReLU(r Wh + bh), take gq = dQp_cache/sqrt(R)
// (the cache stores Qp/sqrt(R)) and gk = dKp_cache, and form
// dpre = (gq Wpq^T + gk Wpk^T) * [pre > 0]. Stores r, h and dpre per token.
__global__ void __launch_bounds__(256) pos_bwd_token_kernel(int M, int L, int hidden, int heads, int R,
                                                            const float* __restrict__ Wh, const float* __restrict__ bh,
                                                            const float* __restrict__ Wpq, const float* __restrict__ Wpk,
                                                            const float* __restrict__ dqp, const float* __restrict__ dkp,
                                                            float q_scale, float* __restrict__ r_out,
                                                            float* __restrict__ h_out, float* __restrict__ dpre_out) {
  __shared__ float r[2 + 4 * 16];
  __shared__ float gq[256], gk[256];
  const int t = blockIdx.x;
  const int i = t / M, j = t % M;
  const int E = 2 + 4 * L;
  const int N = M * M;
  const int outs = heads * R;
  if (threadIdx.x < E) r[threadIdx.x] = fourier_feature(M, i, j, threadIdx.x);   // one thread per feature
  for (int o = threadIdx.x; o < outs; o += blockDim.x) {
    const int hd = o / R, rr = o % R;
    const size_t src = (static_cast<size_t>(hd) * N + t) * R + rr;
    gq[o] = dqp[src] * q_scale;
    gk[o] = dkp[src];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) r_out[static_cast<size_t>(t) * E + e] = r[e];
  // pre-activation, one thread per hidden unit (Wh reads coalesced over k)
  __shared__ float pre[256];
  for (int k = threadIdx.x; k < hidden; k += blockDim.x) {
    float a = __ldg(bh + k);
    for (int e = 0; e < E; ++e) a = fmaf(r[e], __ldg(Wh + e * hidden + k), a);
    pre[k] = a;
    h_out[static_cast<size_t>(t) * hidden + k] = fmaxf(a, 0.f);
  }
  __syncthreads();
  // back through the two output layers: one warp per hidden unit, lanes over
  // the outputs (Wpq/Wpk rows read contiguously), then a warp sum
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int k = warp; k < hidden; k += blockDim.x >> 5) {
    float dh = 0.f;
    for (int o = lane; o < outs; o += 32)
      dh = fmaf(gq[o], __ldg(Wpq + k * outs + o), fmaf(gk[o], __ldg(Wpk + k * outs + o), dh));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dh += __shfl_xor_sync(0xffffffffu, dh, off);
    if (lane == 0) dpre_out[static_cast<size_t>(t) * hidden + k] = pre[k] > 0.f ? dh : 0.f;
  }
}

// Step 2: weight gradients as sums over the window tokens, one thread per
// weight element and token chunk (blockIdx.y), tokens in a fixed order:
//   dWpq[k][o] = sum_t h[t][k] gq[t][o],   dWpk likewise,
//   dWh[e][k]  = sum_t r[t][e] dpre[t][k], dbh[k] = sum_t dpre[t][k].
// Element id: [0, n_p) dWpq, [n_p, 2 n_p) dWpk, then dWh, then dbh; the
// chunk's partial goes to part[chunk][id].
__global__ void pos_bwd_reduce_kernel(int N, int E, int hidden, int heads, int R, const float* __restrict__ r_in,
                                      const float* __restrict__ h_in, const float* __restrict__ dpre_in,
                                      const float* __restrict__ dqp, const float* __restrict__ dkp,
                                      float* __restrict__ part, int total) {
  const int outs = heads * R;
  const int n_p = hidden * outs;
  const int id = blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= total) return;
  const int cs = (N + kPosBwdChunks - 1) / kPosBwdChunks;
  const int t0 = blockIdx.y * cs;
  const int t1 = t0 + cs < N ? t0 + cs : N;
  float acc = 0.f;
  if (id < 2 * n_p) {
    const bool isq = id < n_p;
    const int idx = isq ? id : id - n_p;
    const int k = idx / outs, o = idx % outs;
    const int hd = o / R, rr = o % R;
    const float* g = (isq ? dqp : dkp) + static_cast<size_t>(hd) * N * R + rr;
#pragma unroll 4
    for (int t = t0; t < t1; ++t) acc = fmaf(h_in[static_cast<size_t>(t) * hidden + k], g[static_cast<size_t>(t) * R], acc);
  } else if (id - 2 * n_p < E * hidden) {
    const int id2 = id - 2 * n_p;
    const int e = id2 / hidden, k = id2 % hidden;
#pragma unroll 4
    for (int t = t0; t < t1; ++t) acc = fmaf(r_in[static_cast<size_t>(t) * E + e], dpre_in[static_cast<size_t>(t) * hidden + k], acc);
  } else {
    const int k = id - 2 * n_p - E * hidden;
#pragma unroll 4
    for (int t = t0; t < t1; ++t) acc += dpre_in[static_cast<size_t>(t) * hidden + k];
  }
  part[static_cast<size_t>(blockIdx.y) * total + id] = acc;
}

// Step 3: the chunk partials summed in chunk order into the outputs (dWpq
// takes the cache's 1/sqrt(R) factor).
__global__ void pos_bwd_sum_kernel(int E, int hidden, int heads, int R, const float* __restrict__ part, int total,
                                   float q_scale, float* __restrict__ dWh, float* __restrict__ dbh,
                                   float* __restrict__ dWpq, float* __restrict__ dWpk) {
  const int id = blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= total) return;
  float acc = 0.f;
  for (int c = 0; c < kPosBwdChunks; ++c) acc += part[static_cast<size_t>(c) * total + id];
  const int n_p = hidden * heads * R;
  if (id < n_p) dWpq[id] = acc * q_scale;
  else if (id < 2 * n_p) dWpk[id - n_p] = acc;
  else if (id < 2 * n_p + E * hidden) dWh[id - 2 * n_p] = acc;
  else dbh[id - 2 * n_p - E * hidden] = acc;
}

}  // namespace

cudaError_t launch_pos_encode_bwd(const rib_mlp_desc& m, int M, const float* dqp, const float* dkp, float* dWh,
                                  float* dbh, float* dWpq, float* dWpk, float* ws, cudaStream_t stream) {
  const int N = M * M, E = 2 + 4 * m.L;
  float* r_ws = ws;
  float* h_ws = r_ws + static_cast<size_t>(N) * E;
  float* d_ws = h_ws + static_cast<size_t>(N) * m.hidden;
  const float qs = 1.0f / sqrtf(static_cast<float>(m.R));
  pos_bwd_token_kernel<<<N, 256, 0, stream>>>(M, m.L, m.hidden, m.heads, m.R, m.Wh, m.bh, m.Wpq, m.Wpk, dqp, dkp, qs,
                                              r_ws, h_ws, d_ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int total = 2 * m.hidden * m.heads * m.R + E * m.hidden + m.hidden;
  float* part = d_ws + static_cast<size_t>(N) * m.hidden;
  dim3 grid((total + 127) / 128, kPosBwdChunks);
  pos_bwd_reduce_kernel<<<grid, 128, 0, stream>>>(N, E, m.hidden, m.heads, m.R, r_ws, h_ws, d_ws, dqp, dkp, part, total);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pos_bwd_sum_kernel<<<(total + 127) / 128, 128, 0, stream>>>(E, m.hidden, m.heads, m.R, part, total, qs, dWh, dbh,
                                                               dWpq, dWpk);
  return cudaGetLastError();
}

cudaError_t launch_layernorm(const void* x, int xtype, void* y, int y_f16, long long T, int C, const float* gamma,
                             const float* beta, float eps, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((T * 32 + 255) / 256);
  uint16_t* yb = static_cast<uint16_t*>(y);
  auto kern = y_f16 ? (xtype == 1 ? layernorm_kernel<1, true> : (xtype == 2 ? layernorm_kernel<2, true> : layernorm_kernel<0, true>))
                    : (xtype == 1 ? layernorm_kernel<1, false>
                                  : (xtype == 2 ? layernorm_kernel<2, false> : layernorm_kernel<0, false>));
  kern<<<blocks, 256, 0, stream>>>(x, yb, T, C, gamma, beta, eps);
  return cudaGetLastError();
}

cudaError_t launch_bf16_to_f32(const void* x, float* y, size_t n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const size_t threads = 256;
  const size_t blocks = (n / 4 + threads) / threads;
  bf16_to_f32_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), y, n);
  return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float* x, void* y, size_t n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const size_t threads = 256;
  const size_t blocks = (n / 4 + threads) / threads;
  f32_to_bf16_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(x, static_cast<__nv_bfloat16*>(y), n);
  return cudaGetLastError();
}

cudaError_t launch_pos_encode(const rib_mlp_desc& m, int M, void* qp, void* kp, cudaStream_t stream) {
  const int N = M * M;
  pos_encode_kernel<<<N, 256, 0, stream>>>(M, m.L, m.hidden, m.heads, m.R, m.Wh, m.bh, m.Wpq, m.Wpk,
                                           static_cast<__nv_bfloat16*>(qp), static_cast<__nv_bfloat16*>(kp),
                                           1.0f / sqrtf(static_cast<float>(m.R)));
  return cudaGetLastError();
}

}  // namespace rib
