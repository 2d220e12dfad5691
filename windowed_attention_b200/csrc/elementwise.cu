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

// Steps 1 and 2 in one pass per token chunk, for shapes whose per-thread
// accumulators fit in registers (pos_bwd_chunk_fits). Grid (chunk, output
// group): group 0 accumulates dWpq = sum_t h gq, group 1 dWpk = sum_t h gk,
// group 2 dWh = sum_t r dpre and dbh = sum_t dpre, each over the chunk's
// tokens in order, from r, h (and, for group 2, dpre) recomputed for 32
// tokens at a time in shared memory. The partials go to part[chunk][id] as in
// step 2, summed by step 3.
constexpr int kPbSub = 32;      // tokens per shared-memory sub-tile
constexpr int kPbAcc = 64;      // accumulators per thread at most (dWpq, dWpk)
constexpr int kPbAccE = 32;     // ... (dWh)
constexpr int kPbThreads = 256;
constexpr int kPbChunks = 48;   // token chunks (<= kPosBwdChunks, the workspace's partial slots)
static_assert(kPbChunks <= kPosBwdChunks, "the workspace holds kPosBwdChunks partials");

// shared memory of the chunk kernel: the sub-tile's r, h, gq, gk, dpre (rows
// padded to 4 floats, padding zero) and Wpq^T, Wpk^T (group 2 reads them
// across the hidden units: consecutive threads, consecutive words)
__host__ __device__ inline int pb_pad4(int v) { return (v + 3) & ~3; }
__host__ __device__ inline size_t pos_bwd_chunk_smem(int E, int hidden, int outs, int M) {
  return sizeof(float) * (static_cast<size_t>(kPbSub) * (pb_pad4(E) + 2 * pb_pad4(hidden) + 2 * outs) +
                          2 * static_cast<size_t>(outs) * hidden + static_cast<size_t>(M) * ((E - 2) / 2 + 1));
}
// each thread owns a contiguous run of at most kPbAcc k (groups 0, 1) or e (group 2)
__host__ __device__ inline int pb_kper(int hidden, int outs) { return pb_pad4((hidden + kPbThreads / outs - 1) / (kPbThreads / outs)); }
__host__ __device__ inline int pb_eper(int E, int hidden) { return pb_pad4((E + kPbThreads / hidden - 1) / (kPbThreads / hidden)); }
// hidden = 8 MT: each thread of the token-parallel passes takes MT tokens of
// the 32-token sub-tile (a compile-time count, so their FMA chains are
// unrolled and interleaved)
__host__ __device__ inline bool pos_bwd_chunk_fits(int E, int hidden, int outs, int M) {
  return (hidden == 64 || hidden == 128) && outs % 16 == 0 && outs <= kPbThreads && pb_kper(hidden, outs) <= kPbAcc &&
         pb_eper(E, hidden) <= kPbAccE && pos_bwd_chunk_smem(E, hidden, outs, M) <= 200 * 1024;
}

template <int MT>
__global__ void __launch_bounds__(kPbThreads) pos_bwd_chunk_kernel(
    int M, int L, int hidden, int heads, int R, const float* __restrict__ Wh, const float* __restrict__ bh,
    const float* __restrict__ Wpq, const float* __restrict__ Wpk, const float* __restrict__ dqp,
    const float* __restrict__ dkp, float q_scale, int n_chunks, float* __restrict__ part, int total) {
  extern __shared__ float4 pb_smem4[];
  float* pb_smem = reinterpret_cast<float*>(pb_smem4);
  const int E = 2 + 4 * L, N = M * M, outs = heads * R, n_p = hidden * outs;
  const int Ep = pb_pad4(E), Hp = pb_pad4(hidden);
  const int grp = blockIdx.y;
  float* rs = pb_smem;                       // [kPbSub][Ep]
  float* hs = rs + kPbSub * Ep;              // [kPbSub][Hp]
  float* gqs = hs + kPbSub * Hp;             // [kPbSub][outs] (gq, or gk for group 1)
  float* gks = gqs + kPbSub * outs;          // [kPbSub][outs] (group 2)
  float* ds = gks + kPbSub * outs;           // [kPbSub][Hp] (group 2: dpre)
  float* wqt = ds + kPbSub * Hp;             // [outs][hidden] Wpq^T (group 2)
  float* wkt = wqt + outs * hidden;          // [outs][hidden] Wpk^T (group 2)
  // the encoding is separable: feature e of token (i, j) is a function of the
  // grid coordinate of row i or of column j alone, so the M x (2L + 1) values
  // v, sin(2^b v), cos(2^b v) of the M grid coordinates are evaluated once
  // (in double, as fourier_feature does) and looked up per token
  const int nf = 1 + 2 * L;
  float* tab = wkt + outs * hidden;          // [M][nf]
  const int tid = threadIdx.x;
  const int c = blockIdx.x;
  const int t_begin = static_cast<int>(static_cast<long long>(c) * N / n_chunks);
  const int t_end = static_cast<int>(static_cast<long long>(c + 1) * N / n_chunks);
  // accumulator ownership: groups 0/1 thread = (output o, k run [k0, k0 + kper));
  // group 2 thread = (hidden unit k, e run [e0, e0 + eper))
  const int kgn = kPbThreads / outs, egn = kPbThreads / hidden;
  const int kper = pb_kper(hidden, outs), eper = pb_eper(E, hidden);
  const int o_own = tid % outs, k0 = (tid / outs) * kper;
  const int k_own = tid % hidden, e0 = (tid / hidden) * eper;
  const bool own = grp < 2 ? (tid / outs < kgn && k0 < hidden) : (tid / hidden < egn && e0 < E);
  // token-parallel passes (h, dpre): thread = (hidden unit kk, tokens ig, ig + egn, ...);
  // hidden divides the block, so every thread takes part
  const int kk = tid % hidden, ig = tid / hidden;
  if (grp == 2) {
    for (int x = tid; x < outs * hidden; x += kPbThreads) {
      const int o = x / hidden, k = x - o * hidden;
      wqt[x] = __ldg(Wpq + k * outs + o);
      wkt[x] = __ldg(Wpk + k * outs + o);
    }
  }
  for (int x = tid; x < M * nf; x += kPbThreads) {
    const int i = x / nf, f = x - i * nf;
    // feature 0 of a row (its coordinate), 2 + 4b (sin) and 4 + 4b (cos)
    tab[x] = fourier_feature(M, i, 0, f == 0 ? 0 : (f & 1 ? 2 + 4 * ((f - 1) >> 1) : 4 + 4 * ((f - 2) >> 1)));
  }
  __syncthreads();
  // one sub-tile of tokens [s0, s0 + ns) into shared memory: r, the upstream
  // gradients, h (rows padded with zeros); ends with the block synchronised
  auto subtile = [&](int s0, int ns) {
    for (int x = tid; x < kPbSub * Ep; x += kPbThreads) {
      const int i = x / Ep, e = x - i * Ep, t = s0 + i;
      float v = 0.f;
      if (i < ns && e < E) {
        // e = 0, 1: y, x; e = 2 + 4b + w: sin(2^b y), sin(2^b x), cos(2^b y), cos(2^b x)
        const int w = (e - 2) & 3, b = (e - 2) >> 2;
        const int rc = (e < 2 ? e : (w & 1)) ? t % M : t / M;   // column for x, row for y
        const int f = e < 2 ? 0 : (w < 2 ? 1 + 2 * b : 2 + 2 * b);
        v = tab[rc * nf + f];
      }
      rs[x] = v;
    }
    // upstream gradients: dpre takes the cache's q scale in gq (group 2); the
    // dWpq partials do not (step 3 applies it once, as for the other path)
    for (int x = tid; x < kPbSub * outs; x += kPbThreads) {
      const int i = x / outs, o = x - i * outs;
      float a = 0.f, b = 0.f;
      if (i < ns) {
        const size_t src = (static_cast<size_t>(o / R) * N + s0 + i) * R + (o % R);
        a = grp == 1 ? dkp[src] : dqp[src] * (grp == 2 ? q_scale : 1.f);
        if (grp == 2) b = dkp[src];
      }
      gqs[x] = a;
      if (grp == 2) gks[x] = b;
    }
    __syncthreads();
    // h = ReLU(r Wh + bh): thread = (hidden unit kk, tokens ig + m egn); each
    // weight read once per sub-tile, four e at a time against float4 rows of r
    {
      float a[MT];
      const float b = __ldg(bh + kk);
#pragma unroll
      for (int m = 0; m < MT; ++m) a[m] = b;
      for (int e = 0; e < Ep; e += 4) {
        const float w0 = e < E ? __ldg(Wh + e * hidden + kk) : 0.f;
        const float w1 = e + 1 < E ? __ldg(Wh + (e + 1) * hidden + kk) : 0.f;
        const float w2 = e + 2 < E ? __ldg(Wh + (e + 2) * hidden + kk) : 0.f;
        const float w3 = e + 3 < E ? __ldg(Wh + (e + 3) * hidden + kk) : 0.f;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float4 r4 = *reinterpret_cast<const float4*>(rs + (ig + m * egn) * Ep + e);
          a[m] = fmaf(r4.x, w0, fmaf(r4.y, w1, fmaf(r4.z, w2, fmaf(r4.w, w3, a[m]))));
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int i = ig + m * egn;
        hs[i * Hp + kk] = i < ns ? fmaxf(a[m], 0.f) : 0.f;
      }
    }
    __syncthreads();
  };
  float* pc = part + static_cast<size_t>(c) * total;   // this chunk's partials [dWpq | dWpk | dWh | dbh]
  if (grp == 2) {
    // dWh = sum_t r dpre, dbh = sum_t dpre
    float acc[kPbAccE];
#pragma unroll
    for (int j = 0; j < kPbAccE; ++j) acc[j] = 0.f;
    float acc_b = 0.f;
    for (int s0 = t_begin; s0 < t_end; s0 += kPbSub) {
      const int ns = t_end - s0 < kPbSub ? t_end - s0 : kPbSub;
      subtile(s0, ns);
      // dpre = (gq Wpq^T + gk Wpk^T) * [pre > 0] (pre > 0 exactly where h > 0);
      // separate q and k partial sums keep the dependent chains short
      {
        float dq[MT], dk[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          dq[m] = 0.f;
          dk[m] = 0.f;
        }
        for (int o = 0; o < outs; o += 4) {
          float wq[4], wk[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            wq[q] = wqt[(o + q) * hidden + kk];
            wk[q] = wkt[(o + q) * hidden + kk];
          }
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const int i = ig + m * egn;
            const float4 g4 = *reinterpret_cast<const float4*>(gqs + i * outs + o);
            const float4 k4 = *reinterpret_cast<const float4*>(gks + i * outs + o);
            dq[m] = fmaf(g4.x, wq[0], fmaf(g4.y, wq[1], fmaf(g4.z, wq[2], fmaf(g4.w, wq[3], dq[m]))));
            dk[m] = fmaf(k4.x, wk[0], fmaf(k4.y, wk[1], fmaf(k4.z, wk[2], fmaf(k4.w, wk[3], dk[m]))));
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int i = ig + m * egn;
          ds[i * Hp + kk] = hs[i * Hp + kk] > 0.f ? dq[m] + dk[m] : 0.f;
        }
      }
      __syncthreads();
      if (own) {
        for (int i = 0; i < ns; ++i) {
          const float dk = ds[i * Hp + k_own];
#pragma unroll
          for (int j = 0; j < kPbAccE; j += 4) {
            if (j < eper) {
              const float4 r4 = *reinterpret_cast<const float4*>(rs + i * Ep + e0 + j);
              acc[j] = fmaf(r4.x, dk, acc[j]);
              acc[j + 1] = fmaf(r4.y, dk, acc[j + 1]);
              acc[j + 2] = fmaf(r4.z, dk, acc[j + 2]);
              acc[j + 3] = fmaf(r4.w, dk, acc[j + 3]);
            }
          }
          if (e0 == 0) acc_b += dk;
        }
      }
      __syncthreads();
    }
    if (own) {
#pragma unroll
      for (int j = 0; j < kPbAccE; ++j) {
        const int e = e0 + j;
        if (j < eper && e < E) pc[2 * n_p + e * hidden + k_own] = acc[j];
      }
      if (e0 == 0) pc[2 * n_p + E * hidden + k_own] = acc_b;
    }
  } else {
    // dWpq = sum_t h gq (group 0), dWpk = sum_t h gk (group 1)
    float acc[kPbAcc];
#pragma unroll
    for (int j = 0; j < kPbAcc; ++j) acc[j] = 0.f;
    for (int s0 = t_begin; s0 < t_end; s0 += kPbSub) {
      const int ns = t_end - s0 < kPbSub ? t_end - s0 : kPbSub;
      subtile(s0, ns);
      if (own) {
        for (int i = 0; i < ns; ++i) {
          const float g = gqs[i * outs + o_own];
#pragma unroll
          for (int j = 0; j < kPbAcc; j += 4) {
            if (j < kper) {
              const float4 h4 = *reinterpret_cast<const float4*>(hs + i * Hp + k0 + j);
              acc[j] = fmaf(h4.x, g, acc[j]);
              acc[j + 1] = fmaf(h4.y, g, acc[j + 1]);
              acc[j + 2] = fmaf(h4.z, g, acc[j + 2]);
              acc[j + 3] = fmaf(h4.w, g, acc[j + 3]);
            }
          }
        }
      }
      __syncthreads();
    }
    if (own) {
#pragma unroll
      for (int j = 0; j < kPbAcc; ++j) {
        const int k = k0 + j;
        if (j < kper && k < hidden) pc[grp * n_p + k * outs + o_own] = acc[j];
      }
    }
  }
}

// Step 3: the chunk partials summed in chunk order into the outputs (dWpq
// takes the cache's 1/sqrt(R) factor).
__global__ void pos_bwd_sum_kernel(int E, int hidden, int heads, int R, const float* __restrict__ part, int total,
                                   int n_chunks, float q_scale, float* __restrict__ dWh, float* __restrict__ dbh,
                                   float* __restrict__ dWpq, float* __restrict__ dWpk) {
  const int id = blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= total) return;
  float acc = 0.f;
  for (int c = 0; c < n_chunks; ++c) acc += part[static_cast<size_t>(c) * total + id];
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
  const int total = 2 * m.hidden * m.heads * m.R + E * m.hidden + m.hidden;
  float* part = d_ws + static_cast<size_t>(N) * m.hidden;
  if (pos_bwd_chunk_fits(E, m.hidden, m.heads * m.R, M)) {
    const int outs = m.heads * m.R;
    const size_t smem = pos_bwd_chunk_smem(E, m.hidden, outs, M);
    auto kern = m.hidden == 128 ? pos_bwd_chunk_kernel<16> : pos_bwd_chunk_kernel<8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // one wave: 48 chunks x 3 output groups, one CTA per SM (the
    // accumulators take the register file)
    const int n_chunks = N < kPbChunks ? N : kPbChunks;
    kern<<<dim3(n_chunks, 3), kPbThreads, smem, stream>>>(M, m.L, m.hidden, m.heads, m.R, m.Wh, m.bh, m.Wpq, m.Wpk, dqp,
                                                          dkp, qs, n_chunks, part, total);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    pos_bwd_sum_kernel<<<(total + 127) / 128, 128, 0, stream>>>(E, m.hidden, m.heads, m.R, part, total, n_chunks, qs,
                                                                 dWh, dbh, dWpq, dWpk);
    return cudaGetLastError();
  }
  pos_bwd_token_kernel<<<N, 256, 0, stream>>>(M, m.L, m.hidden, m.heads, m.R, m.Wh, m.bh, m.Wpq, m.Wpk, dqp, dkp, qs,
                                              r_ws, h_ws, d_ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid((total + 127) / 128, kPosBwdChunks);
  pos_bwd_reduce_kernel<<<grid, 128, 0, stream>>>(N, E, m.hidden, m.heads, m.R, r_ws, h_ws, d_ws, dqp, dkp, part, total);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pos_bwd_sum_kernel<<<(total + 127) / 128, 128, 0, stream>>>(E, m.hidden, m.heads, m.R, part, total, kPosBwdChunks,
                                                               qs, dWh, dbh, dWpq, dWpk);
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
