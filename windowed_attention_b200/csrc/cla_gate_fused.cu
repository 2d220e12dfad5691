// Fused depthwise 3x3 -> pointwise kernel, used for two steps of the SST
// block (RIB/SST write-up):
//  * the CLA gate, sigmoid(PWConv(DWConv3x3(X))) in one pass over X (section
//    2.3: G = PWConv(DWConv3x3(X)), applied as sigmoid(G));
//  * the second half of the ConvFFN (section 3.1): with h the GELU hidden
//    features, x += (h + DWConv3x3(h)) W2 + b2 into the fp32 residual stream;
//    the inner residual h is the depthwise filter's centre tap plus one. Here
//    h, the depthwise tile and W2 are fp16 (the hidden features of a
//    LayerNorm-ed input are bounded; fp16 keeps 4x finer steps than bf16, and
//    the conversions saturate).
//
// Written below for the gate (C input and output channels); the ConvFFN
// differs in the channel counts (Cin hidden channels padded to 8, of which
// the first Cw carry weights; Cout = C outputs) and the epilogue.
// Per output tile of 4 rows x 16 columns (64 pixels) of one image:
//   D[p][c] = bdw[c] + sum_{dy,dx} Wdw[c][dy][dx] X[p + (dy-1, dx-1)][c]   (zero padding 1)
//   G[p][n] = bpw[n] + sum_c D[p][c] Wpw[c][n],     out[p][n] = bf16(sigmoid(G[p][n]))
// without D ever reaching global memory (unless the caller asks for it, for
// the backward).
//
// Data movement. X is read through a TMA tensor map that views each image row
// as W*C/L lines of L elements (L = 256, 128, ..., 8, the widest dividing W*C:
// the TMA moves a box row by row, so long lines cost fewer transfers):
// channels-last pixels of C bf16 are 2C bytes apart, which need not be a
// multiple of 16, but a row of lines is. One box per (input row, part of the
// row) brings the tile's 6 input rows x 18 pixels (the 3x3 halo) into shared
// memory as contiguous runs of elements;
// rows above/below the image and chunks left/right of it are zero-filled by
// the TMA, which is exactly the convolution's zero padding. Two input stages.
//
// Depthwise. Nine warps (gate) or six (ConvFFN) compute D in fp32 (packed
// pairs of channels), thread = 4 channels x every dlanes-th column of the
// tile (dlanes = depthwise threads / channel groups, at most 16), sliding
// down the tile's 4 output rows, and write it as bf16 into the
// 128-byte-swizzled K-major operand tile [64 pixels][K = C padded to 64] in
// shared memory (two stages).
//
// Pointwise. The transposed product G^T = Wpw^T D^T runs on tcgen05 with
// Wpw^T as the A operand held in TMEM for the CTA's lifetime (loaded once)
// and the D tile as the B operand: M = 128 output channels per MMA (a second
// MMA covers channels C-128 .. C-1 when C > 128), N = 64 pixels, K = C padded.
// The fp32 accumulator sits in TMEM with output channels in lanes, two
// accumulator stages. The two halves' MMAs go out from two threads: one
// thread issues an M = 128, K = 16 product about every 55 cycles at N <= 64,
// while the SM retires one every ~48 cycles at N = 64, so a second issuing
// thread is what reaches the SM's rate.
//
// Epilogue. Four warps (gate) or eight (ConvFFN: two per TMEM lane quarter,
// one per 32-pixel half of the tile), thread = output channel: bias, sigmoid (tanh.approx),
// bf16 into a shared-memory staging tile [64 pixels][Cout] (each warp store
// writes 32 consecutive channels), then one bulk copy per tile row (16 pixels
// x Cout, contiguous in the channels-last output); two staging buffers, so a
// tile's copies overlap the next tile's epilogue. The ConvFFN epilogue adds
// into the fp32 residual stream directly (each warp access 32 consecutive
// channels, 128 bytes).
//
// Warp roles: 0 TMA producer (and, in the ConvFFN, the second half's MMA
// issuer), 1 MMA issuer and TMEM owner, 2 .. DW + 1 depthwise, then NEPI
// epilogue warps, then (gate with C > 128) one warp issuing the second
// half's MMAs. Persistent grid, one CTA per SM (the CTA holds all 512 TMEM
// columns).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "rib_internal.h"
#include "sm100.cuh"

namespace rib {

namespace {

constexpr int kTY = 4, kTX = 16, kTP = kTY * kTX;   // output tile: 4 rows x 16 columns
constexpr int kInRows = kTY + 2;                      // input rows of a tile (halo)
// NEPI epilogue warps: 4 (one per TMEM lane quarter, the gate) or 8 (two
// per quarter, one per 32-pixel half: the ConvFFN, whose fp32
// read-modify-write epilogue is the slower one)
// X2: one more warp after the epilogue warps, the second output half's MMA
// issuer (the gate: its own instruction stream, waiting on nothing but the
// tiles' barriers)
// DW: depthwise warps (2 .. DW + 1), then the epilogue warps from 2 + DW
template <int NEPI, int X2, int DW>
__host__ __device__ constexpr int threads_of() { return (2 + DW + NEPI + X2) * 32; }
constexpr int kMaxIn = 3;                             // input stages at most
constexpr int kAccCols = 128;                         // one accumulator stage: two M=128 x N=64 tiles

enum FusedGateSite : int {
  SITE_F_IN_FREE = 401, SITE_F_IN_FULL = 402, SITE_F_D_FREE = 403, SITE_F_D_FULL = 404,
  SITE_F_ACC_FREE = 405, SITE_F_ACC_FULL = 406, SITE_F_DRAIN = 407,
};

struct FusedGateParams {
  int B, H, W;
  int C;             // input channels of the map the TMA reads (Cin)
  int Cw;            // input channels with depthwise weights and pointwise rows (<= C; the rest are zero)
  int Cout;          // output channels
  int ffn;           // 0: gate epilogue (sigmoid, bf16 out); 1: ConvFFN epilogue (+ bias into fp32 xres), fp16 product
  int x_f16;         // the map read by the TMA is fp16 (else bf16)
  int KA;            // 64-channel K atoms of the padded reduction
  int two_m;         // C > 128: a second MMA covers output channels c2 .. c2 + 127
  int c2;
  int tiles_x, tiles_y, n_tiles;
  int L;             // elements per TMA line (256 .. 8: the widest dividing W*C)
  int nbox, bc;      // TMA boxes per input row and lines per box
  int row_bytes;     // bytes of one input row in shared memory (nbox * bc * L * 2)
  int in_stage;      // bytes of one input stage
  int d_stage;       // bytes of one D tile stage (KA * 64 * 128)
  int off_d, off_st, off_misc;   // shared memory: input stages | D stages | output staging (gate) | barriers
  int st_bytes;      // gate: one output staging buffer, [64 pixels][Cout] bf16
  int nst;           // gate: staging buffers (2, or 1 when two do not fit)
  int split;         // two output halves issued from two threads: warp 1 and 1 = the producer, 2 = an extra warp
  int dlanes;        // depthwise threads per channel group (columns handled in parallel)
  int nin;           // input stages (2 or 3, as shared memory allows)
  const float* Wdw;  // [C][3][3]
  const float* bdw;  // [C]
  const __nv_bfloat16* Wpw;   // [C][C] (in, out)
  const float* bpw;  // [C]
  __nv_bfloat16* out;         // gate: [B][H][W][Cout]
  __nv_bfloat16* D_out;       // gate, optional: the depthwise output [B][H][W][C]
  float* xres;                // ConvFFN: the fp32 residual stream [B][H][W][Cout], updated in place
  int* err;
};

__device__ __forceinline__ float sigmoid_tanh(float v) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * v));
  return fmaf(0.5f, t, 0.5f);
}

__device__ __forceinline__ bool warp_all_f(bool v) { return __all_sync(0xffffffffu, v); }

__device__ __forceinline__ void bulk_store(void* gdst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               ::"l"(reinterpret_cast<uint64_t>(gdst)), "r"(smem_u32(src)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// named barrier 1: the NEPI epilogue warps
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

template <int NEPI, int X2, int DW>
__global__ void __launch_bounds__(threads_of<NEPI, X2, DW>(), 1)
cla_gate_fused_kernel(const __grid_constant__ CUtensorMap tm_x, const FusedGateParams p) {
  constexpr int kThreads = threads_of<NEPI, X2, DW>();
  constexpr int kDWarps = DW;
  constexpr int kEpi0 = 2 + DW;   // first epilogue warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* s_in = smem;                    // two input stages
  uint8_t* s_d = smem + p.off_d;           // two D tile stages (1024-byte aligned)
  uint8_t* s_st = smem + p.off_st;         // gate: two output staging buffers
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_misc);
  uint64_t* in_full = bars;                  // [kMaxIn]
  uint64_t* in_free = bars + kMaxIn;         // [kMaxIn]
  uint64_t* d_full = bars + 2 * kMaxIn;      // [2]
  uint64_t* d_free = d_full + 2;             // [2]
  uint64_t* acc_full = d_full + 4;           // [2]
  uint64_t* acc_free = d_full + 6;           // [2]
  uint64_t* done = d_full + 8;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(d_full + 9);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(tmem_holder + 1);

  if (tid == 0) {
    for (int i = 0; i < kMaxIn; ++i) {
      mbar_init(&in_full[i], 1);
      mbar_init(&in_free[i], kDWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&d_full[i], kDWarps);
      // with two output halves (C > 128) two threads issue the MMAs of a tile
      mbar_init(&d_free[i], p.split ? 2 : 1);
      mbar_init(&acc_full[i], p.split ? 2 : 1);
      mbar_init(&acc_free[i], NEPI);
    }
    mbar_init(done, p.split ? 2 : 1);
    *abort_flag = 0u;
    tmem_holder[2] = 0u;   // abort word of the teardown drains (never raised)
    fence_barrier_init();
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  // zero both D stages: the K padding (channels C .. 64 KA - 1) stays zero
  for (int i = tid; i < 2 * p.d_stage / 16; i += kThreads)
    reinterpret_cast<uint4*>(s_d)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int acol = p.KA * 32;   // TMEM columns of one A operand (K/2 bf16 pairs)

  // Wpw^T into TMEM (A operands): lane = output channel, column k/2 = input
  // channels (k, k+1) as a bf16 pair; channels past C are zero.
  if (warp >= kEpi0 && warp < kEpi0 + 4) {
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    for (int m = 0; m < 1 + p.two_m; ++m) {
      const int n = (m == 0 ? 0 : p.c2) + q * 32 + lane;   // output channel of this lane
      for (int a = 0; a < p.KA; ++a) {                      // 32 columns = 64 input channels
        uint32_t v[32];
#pragma unroll 4
        for (int i = 0; i < 32; ++i) {   // (set-up only: partly unrolled to spare registers)
          const int k = a * 64 + 2 * i;
          const uint16_t* W = reinterpret_cast<const uint16_t*>(p.Wpw);
          const uint32_t lo = (n < p.Cout && k < p.Cw) ? __ldg(W + static_cast<size_t>(k) * p.Cout + n) : 0u;
          const uint32_t hi = (n < p.Cout && k + 1 < p.Cw) ? __ldg(W + static_cast<size_t>(k + 1) * p.Cout + n) : 0u;
          // the ConvFFN's product runs in fp16: the bf16 weights converted (exact in fp16's normal range)
          v[i] = p.ffn ? pack_f16x2_sat(__uint_as_float(lo << 16), __uint_as_float(hi << 16)) : (lo | (hi << 16));
        }
        tmem_st32(tmem + lane_off + m * acol + a * 32, v);
      }
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const WaitCtx wc{abort_flag, p.err};
  const WaitCtx drain{reinterpret_cast<volatile uint32_t*>(tmem_holder + 2), p.err};

  // MMAs of output half m (channels m == 0 ? 0.. : c2..) of tile iteration it
  const uint32_t idesc = p.ffn ? idesc_f16(128, kTP, false, false) : idesc_bf16(128, kTP, false, false);
  auto issue_half = [&](int it, int m) {
    const int s = it & 1;
    const uint32_t db = smem_u32(s_d) + s * p.d_stage;
    const uint32_t acc = tmem + 256u + s * kAccCols + m * kTP;
    const uint32_t a = tmem + m * acol;
    for (int ks = 0; ks < p.KA * 4; ++ks) {
      // K step ks: atom ks/4, 32-byte offset (ks%4) inside the 128-byte row
      const uint32_t kb = (ks >> 2) * (kTP * 128) + (ks & 3) * 32;
      umma_ts(acc, a + 8u * ks, make_sdesc(db + kb, 16, 1024, SW_128B), idesc, ks > 0 ? 1u : 0u);
    }
  };
  auto release = [&](int it) {
    umma_commit(&d_free[it & 1]);
    umma_commit(&acc_full[it & 1]);
  };
  // waits of tile iteration it's MMAs: its D tile written, its accumulator
  // stage drained by the epilogue of iteration it - 2
  auto mma_ready = [&](int it) {
    const int s = it & 1;
    if (!mbar_wait(&d_full[s], (it >> 1) & 1, wc, SITE_F_D_FULL)) return false;
    if (it >= 2 && !mbar_wait(&acc_free[s], ((it >> 1) - 1) & 1, wc, SITE_F_ACC_FREE)) return false;
    tc_fence_after();
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // (and, with two output halves, the issuer of the second half's MMAs:
    // a second issuing thread reaches the SM's MMA rate, which one thread
    // alone does not; tile it - 2's second half goes out right
    // after tile it's loads, when its depthwise has finished)
    if (lane == 0) {
      int it = 0, issued = 0, mb = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++it) {
        const int s = it % p.nin, ui = it / p.nin;   // input stage and its earlier uses
        if (ui > 0 && !(ok = mbar_wait(&in_free[s], (ui - 1) & 1, wc, SITE_F_IN_FREE))) break;
        const int tx = tile % p.tiles_x, t2 = tile / p.tiles_x;
        const int ty = t2 % p.tiles_y, b = t2 / p.tiles_y;
        const int x0 = tx * kTX, y0 = ty * kTY;
        // first line of the row segment holding pixels x0-1 .. x0+16 (floor division)
        const long long e0 = static_cast<long long>(x0 - 1) * p.C;
        const int k0 = static_cast<int>(e0 >= 0 ? e0 / p.L : -((-e0 + p.L - 1) / p.L));
        mbar_arrive_expect_tx(&in_full[s], static_cast<uint32_t>(p.in_stage));
        uint8_t* dst = s_in + s * p.in_stage;
        for (int r = 0; r < kInRows; ++r)
          for (int k = 0; k < p.nbox; ++k)
            tma_load_4d(dst + r * p.row_bytes + k * p.bc * p.L * 2, &tm_x, &in_full[s], 0, k0 + k * p.bc, y0 - 1 + r, b);
        issued = it + 1;
        if (p.split == 1 && it >= 2) {
          if (!(ok = mma_ready(mb))) break;
          issue_half(mb, 1);
          release(mb++);
        }
      }
      if (p.split == 1) {
        for (; ok && mb < issued; ++mb) {
          if (!(ok = mma_ready(mb))) break;
          issue_half(mb, 1);
          release(mb);
        }
        umma_commit(done);
      }
      for (int i = issued - p.nin > 0 ? issued - p.nin : 0; i < issued; ++i)
        mbar_wait(&in_full[i % p.nin], (i / p.nin) & 1, drain, SITE_F_DRAIN);
      if (p.split == 1) mbar_wait(done, 0, drain, SITE_F_DRAIN);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (first output half)
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++it) {
        if (!mma_ready(it)) break;
        issue_half(it, 0);
        if (p.two_m && !p.split) issue_half(it, 1);
        release(it);
      }
      umma_commit(done);
      mbar_wait(done, 0, drain, SITE_F_DRAIN);
    }
  } else if (warp < kEpi0) {
    // ------------------------------------------------------------ depthwise
    const int t = tid - 64;                      // 0 .. 32 DW - 1
    const int G = p.C / 4;                       // channel groups of 4
    const int g = t % G, xl = t / G;             // group, first column of this thread
    const bool active = xl < p.dlanes;
    // this thread's taps and bias, as packed channel pairs (c, c+1) and (c+2, c+3)
    uint64_t w01[9], w23[9];
    uint64_t b01 = 0, b23 = 0;
    if (active) {
      const int c = 4 * g;
      // channels past Cw carry no weights; the ConvFFN's inner residual h is
      // one more on the centre tap
      auto tap = [&](int cc, int tp) {
        return (cc < p.Cw ? __ldg(p.Wdw + cc * 9 + tp) : 0.f) + ((p.ffn && tp == 4) ? 1.f : 0.f);
      };
      auto bias = [&](int cc) { return cc < p.Cw ? __ldg(p.bdw + cc) : 0.f; };
#pragma unroll
      for (int tp = 0; tp < 9; ++tp) {
        w01[tp] = f2_pack(tap(c + 0, tp), tap(c + 1, tp));
        w23[tp] = f2_pack(tap(c + 2, tp), tap(c + 3, tp));
      }
      b01 = f2_pack(bias(c), bias(c + 1));
      b23 = f2_pack(bias(c + 2), bias(c + 3));
    }
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++it) {
      const int s = it & 1;                        // D stage
      const int si = it % p.nin;                   // input stage
      if (!(ok = warp_all_f(mbar_wait(&in_full[si], (it / p.nin) & 1, wc, SITE_F_IN_FULL)))) break;
      if (it >= 2 && !(ok = warp_all_f(mbar_wait(&d_free[s], ((it >> 1) - 1) & 1, wc, SITE_F_D_FREE)))) break;
      const int tx = tile % p.tiles_x, t2 = tile / p.tiles_x;
      const int ty = t2 % p.tiles_y, b = t2 / p.tiles_y;
      const int x0 = tx * kTX, y0 = ty * kTY;
      const long long e0 = static_cast<long long>(x0 - 1) * p.C;
      const long long k0 = e0 >= 0 ? e0 / p.L : -((-e0 + p.L - 1) / p.L);
      const uint8_t* in = s_in + si * p.in_stage;
      uint8_t* dt = s_d + s * p.d_stage;
      if (active) {
        for (int x = xl; x < kTX; x += p.dlanes) {
          // input columns x-1, x, x+1 of rows 0..5 (element offset in the row
          // segment); each input row is converted once and added into the (up
          // to three) output rows whose 3x3 window contains it
          const int eo = static_cast<int>(static_cast<long long>(x0 + x - 1) * p.C + 4 * g - p.L * k0);
          uint64_t a01[kTY], a23[kTY];
#pragma unroll
          for (int yo = 0; yo < kTY; ++yo) {
            a01[yo] = b01;
            a23[yo] = b23;
          }
#pragma unroll
          for (int r = 0; r < kInRows; ++r) {
            uint64_t i01[3], i23[3];
#pragma unroll
            for (int dx = 0; dx < 3; ++dx) {
              const uint2 u = *reinterpret_cast<const uint2*>(in + r * p.row_bytes + 2 * (eo + dx * p.C));
              if (p.x_f16) {   // fp16 map (the ConvFFN's hidden features, or an fp16 gate input)
                i01[dx] = f2_pack(f16_lo(u.x), f16_hi(u.x));
                i23[dx] = f2_pack(f16_lo(u.y), f16_hi(u.y));
              } else {
                i01[dx] = f2_pack(bf16_lo(u.x), bf16_hi(u.x));
                i23[dx] = f2_pack(bf16_lo(u.y), bf16_hi(u.y));
              }
            }
#pragma unroll
            for (int dy = 0; dy < 3; ++dy) {
              const int yo = r - dy;
              if (yo >= 0 && yo < kTY) {
#pragma unroll
                for (int dx = 0; dx < 3; ++dx) {
                  a01[yo] = f2_fma(w01[dy * 3 + dx], i01[dx], a01[yo]);
                  a23[yo] = f2_fma(w23[dy * 3 + dx], i23[dx], a23[yo]);
                }
              }
            }
          }
#pragma unroll
          for (int yo = 0; yo < kTY; ++yo) {
            float d0, d1, d2, d3;
            f2_unpack(a01[yo], d0, d1);
            f2_unpack(a23[yo], d2, d3);
            const uint2 dv = p.ffn ? make_uint2(pack_f16x2_sat(d0, d1), pack_f16x2_sat(d2, d3))
                                   : make_uint2(pack_bf16x2(d0, d1), pack_bf16x2(d2, d3));
            // operand tile: row px, K = 4g: atom k/64, 16-byte chunk ((k%64)/8) ^ (px%8), half (k%8)/4
            const int px = yo * kTX + x, k = 4 * g;
            *reinterpret_cast<uint2*>(dt + (k >> 6) * (kTP * 128) + px * 128 + ((((k & 63) >> 3) ^ (px & 7)) << 4) +
                                      ((k & 7) >> 2) * 8) = dv;
            if (p.D_out) {
              const int y = y0 + yo, xx = x0 + x;
              if (y < p.H && xx < p.W)
                *reinterpret_cast<uint2*>(p.D_out + ((static_cast<size_t>(b) * p.H + y) * p.W + xx) * p.C + k) = dv;
            }
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&d_full[s]);
        mbar_arrive(&in_free[si]);
      }
    }
  } else if (X2 && warp == kEpi0 + NEPI) {
    // ------------------------------------------------------------ MMA issuer (second output half)
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++it) {
        if (!mma_ready(it)) break;
        issue_half(it, 1);
        release(it);
      }
      umma_commit(done);
      mbar_wait(done, 0, drain, SITE_F_DRAIN);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int hh = (warp - kEpi0) >> 2;           // NEPI == 8: pixels 32 hh .. 32 hh + 31 of each tile
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const int n1 = q * 32 + lane;                 // output channel of this lane in the first MMA
    const int n2 = p.c2 + q * 32 + lane;          // ... and in the second
    const bool st1 = n1 < p.Cout && n1 < 128;
    const bool st2 = p.two_m && n2 >= 128 && n2 < p.Cout;
    const bool warp2 = p.two_m && (p.c2 + q * 32 + 31 >= 128);   // some lane of this warp stores from the second
    const float bias1 = st1 ? __ldg(p.bpw + n1) : 0.f;
    const float bias2 = st2 ? __ldg(p.bpw + n2) : 0.f;
    const bool leader = warp == kEpi0 && lane == 0;   // issues the gate's bulk stores
    int it = 0;
    for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++it) {
      const int s = it & 1;
      if (!warp_all_f(mbar_wait(&acc_full[s], (it >> 1) & 1, wc, SITE_F_ACC_FULL))) break;
      tc_fence_after();
      const int tx = tile % p.tiles_x, t2 = tile / p.tiles_x;
      const int ty = t2 % p.tiles_y, b = t2 / p.tiles_y;
      const int x0 = tx * kTX, y0 = ty * kTY;
      const int nx = p.W - x0 < kTX ? p.W - x0 : kTX;   // columns of the tile inside the image
      const int sb = p.nst == 2 ? s : 0;
      uint16_t* stg = reinterpret_cast<uint16_t*>(s_st + sb * p.st_bytes);
      if (!p.ffn) {
        // the bulk stores issued earlier from this staging buffer have read it
        if (leader) {
          if (p.nst == 2) bulk_wait_read1();
          else bulk_wait_read0();
        }
        named_sync(1, NEPI * 32);
      }
      for (int m = 0; m < 2; ++m) {
        if (m == 1 && !warp2) break;
        const bool st = m == 0 ? st1 : st2;
        const int n = m == 0 ? n1 : n2;
        const float bias = m == 0 ? bias1 : bias2;
        const uint32_t acc = tmem + lane_off + 256u + s * kAccCols + m * kTP;
#pragma unroll 1
        for (int h = NEPI == 8 ? hh : 0; h < (NEPI == 8 ? hh + 1 : kTP / 32); ++h) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(acc + 32 * h, v);
          tmem_wait_ld();
          if (st && p.ffn) {
#pragma unroll
            for (int rr = 0; rr < 32 / kTX; ++rr) {   // the two tile rows of these 32 pixels
              const int y = y0 + (32 / kTX) * h + rr;
              if (y < p.H) {
                float* rp = p.xres + ((static_cast<size_t>(b) * p.H + y) * p.W + x0) * p.Cout + n;
#pragma unroll
                for (int i = 0; i < kTX; ++i)
                  if (i < nx) rp[static_cast<size_t>(i) * p.Cout] += __uint_as_float(v[rr * kTX + i]) + bias;
              }
            }
          } else if (st) {
#pragma unroll
            for (int i = 0; i < 32; ++i)   // pixel 32 h + i of the tile
              stg[(32 * h + i) * p.Cout + n] =
                  static_cast<uint16_t>(pack_bf16x2(sigmoid_tanh(__uint_as_float(v[i]) + bias), 0.f) & 0xFFFFu);
          }
        }
      }
      __syncwarp();
      // accumulator drained: the MMAs of tile it + 2 may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_free[s]);
      if (!p.ffn) {
        fence_proxy_async_smem();
        named_sync(1, NEPI * 32);
        if (leader) {
          const uint32_t row_bytes = static_cast<uint32_t>(nx * p.Cout * 2);
          for (int yo = 0; yo < kTY; ++yo) {
            const int y = y0 + yo;
            if (y < p.H)
              bulk_store(p.out + ((static_cast<size_t>(b) * p.H + y) * p.W + x0) * p.Cout,
                         s_st + sb * p.st_bytes + yo * kTX * p.Cout * 2, row_bytes);
          }
          bulk_commit();
        }
      }
    }
    if (leader) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool dw_pw_fused_supported(const void* X, int W, int Cin, int Cout) {
  return (reinterpret_cast<uintptr_t>(X) % 16) == 0 && Cin % 4 == 0 && Cin >= 4 && Cin <= 256 && Cout >= 1 &&
         Cout <= 256 && (static_cast<long long>(W) * Cin) % 8 == 0;
}

bool cla_gate_fused_supported(const void* X, int B, int H, int W, int C) {
  (void)B;
  (void)H;
  return dw_pw_fused_supported(X, W, C, C);
}

cudaError_t launch_dw_pw_fused(const void* X, int B, int H, int W, int Cin, int Cw, int Cout, const float* Wdw,
                               const float* bdw, const void* Wpw, const float* bpw, void* out, void* D_out, float* xres,
                               int ffn, int x_f16, cudaStream_t stream) {
  FusedGateParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = B;
  p.H = H;
  p.W = W;
  p.C = Cin;
  p.Cw = Cw;
  p.Cout = Cout;
  p.ffn = ffn;
  p.x_f16 = x_f16;
  p.KA = (Cin + 63) / 64;
  p.two_m = Cout > 128 ? 1 : 0;
  // two output halves: a second MMA-issuing thread (the producer in the
  // ConvFFN; in the gate an extra warp, whose stream waits on nothing else)
#ifndef RIB_GATE_X2
#define RIB_GATE_X2 1
#endif
  p.split = p.two_m ? (ffn ? 1 : (RIB_GATE_X2 ? 2 : 0)) : 0;
  p.c2 = Cout > 128 ? Cout - 128 : 0;
  p.tiles_x = (W + kTX - 1) / kTX;
  p.tiles_y = (H + kTY - 1) / kTY;
  const long long tiles = static_cast<long long>(B) * p.tiles_x * p.tiles_y;
  if (tiles == 0) return cudaSuccess;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  p.n_tiles = static_cast<int>(tiles);
  // lines of L elements covering pixels x0-1 .. x0+16 of a row from a
  // line-aligned start: L the widest of 64, 32, 16, 8 dividing W*Cin (fewer,
  // longer TMA lines); boxes of whole multiples of 128 bytes, so every box
  // lands on a 128-byte boundary of shared memory, as tensor copies require
  const long long wc = static_cast<long long>(W) * Cin;
  p.L = 8;
  for (int l = 256; l > 8; l /= 2)
    if (wc % l == 0) {
      p.L = l;
      break;
    }
  const int lines = (18 * Cin + 2 * p.L - 1) / p.L;
  const int align = p.L >= 64 ? 1 : 64 / p.L;   // lines per 128 bytes
  p.nbox = (lines + 255) / 256;
  p.bc = ((lines + p.nbox - 1) / p.nbox + align - 1) / align * align;
  if (p.bc > 256) return cudaErrorInvalidConfiguration;
  p.row_bytes = p.nbox * p.bc * p.L * 2;
  p.in_stage = kInRows * p.row_bytes;
  p.d_stage = p.KA * kTP * 128;
  auto up = [](int v, int a) { return (v + a - 1) / a * a; };
  // input stages | D stages | staging | barriers: three input stages where they
  // fit (the TMA loads' latency is about a tile's depthwise), else two; two
  // staging buffers where they fit, else one
  const int misc_bytes = 24 * 8;
  p.nin = 2;
  p.nst = 1;
  {
    const int stb = ffn ? 0 : up(kTP * Cout * 2, 128);
    const int cfg[4][2] = {{3, 2}, {2, 2}, {3, 1}, {2, 1}};
    for (int i = 0; i < 4; ++i) {
      const int tot = up(cfg[i][0] * p.in_stage, 1024) + 2 * p.KA * kTP * 128 + cfg[i][1] * stb + misc_bytes + 1024;
      if (tot <= 227 * 1024) {
        p.nin = cfg[i][0];
        p.nst = cfg[i][1];
        break;
      }
    }
  }
  p.off_d = up(p.nin * p.in_stage, 1024);
  p.st_bytes = ffn ? 0 : up(kTP * Cout * 2, 128);
  p.off_st = p.off_d + 2 * p.d_stage;
  p.off_misc = p.off_st + p.nst * p.st_bytes;
  const int total = p.off_misc + misc_bytes + 1024;
  if (total > 227 * 1024) return cudaErrorInvalidConfiguration;
  // depthwise warps: nine for the gate (16 warps in all, 128 registers a
  // thread), six for the ConvFFN, whose eight epilogue warps need the rest
  const int dw_threads = (ffn ? 6 : 9) * 32;
  const int G = Cin / 4;
  p.dlanes = dw_threads / G < kTX ? dw_threads / G : kTX;
  if (p.dlanes < 1) return cudaErrorInvalidConfiguration;
  p.Wdw = Wdw;
  p.bdw = bdw;
  p.Wpw = static_cast<const __nv_bfloat16*>(Wpw);
  p.bpw = bpw;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.D_out = static_cast<__nv_bfloat16*>(D_out);
  p.xres = xres;
  p.err = device_error_word();

  // X as [B][H][W*Cin/L lines][L elements]
  CUtensorMap tm;
  const uint64_t dims[4] = {static_cast<uint64_t>(p.L), static_cast<uint64_t>(wc / p.L), static_cast<uint64_t>(H),
                            static_cast<uint64_t>(B)};
  const uint64_t strides[3] = {static_cast<uint64_t>(p.L) * 2, static_cast<uint64_t>(wc) * 2,
                               static_cast<uint64_t>(H) * wc * 2};
  const uint32_t box[4] = {static_cast<uint32_t>(p.L), static_cast<uint32_t>(p.bc), 1u, 1u};
  if (encode_tiled(&tm, x_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(X),
                   dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int grid = p.n_tiles < sm_count() ? p.n_tiles : sm_count();
  if (ffn) {
    cudaError_t e = cudaFuncSetAttribute(cla_gate_fused_kernel<8, 0, 6>, cudaFuncAttributeMaxDynamicSharedMemorySize, total);
    if (e != cudaSuccess) return e;
    cla_gate_fused_kernel<8, 0, 6><<<grid, threads_of<8, 0, 6>(), total, stream>>>(tm, p);
  } else if (p.split == 2) {
    cudaError_t e = cudaFuncSetAttribute(cla_gate_fused_kernel<4, 1, 9>, cudaFuncAttributeMaxDynamicSharedMemorySize, total);
    if (e != cudaSuccess) return e;
    cla_gate_fused_kernel<4, 1, 9><<<grid, threads_of<4, 1, 9>(), total, stream>>>(tm, p);
  } else {
    cudaError_t e = cudaFuncSetAttribute(cla_gate_fused_kernel<4, 0, 9>, cudaFuncAttributeMaxDynamicSharedMemorySize, total);
    if (e != cudaSuccess) return e;
    cla_gate_fused_kernel<4, 0, 9><<<grid, threads_of<4, 0, 9>(), total, stream>>>(tm, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_cla_gate_fused(const void* X, int x_f16, const float* Wdw, const float* bdw, const void* Wpw,
                                  const float* bpw, void* out, void* D_out, int B, int H, int W, int C, cudaStream_t stream) {
  return launch_dw_pw_fused(X, B, H, W, C, C, C, Wdw, bdw, Wpw, bpw, out, D_out, nullptr, 0, x_f16, stream);
}

}  // namespace rib
