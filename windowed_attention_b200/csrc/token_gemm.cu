// Token GEMM on tcgen05: out[t, n] = epilogue( sum_k A[t, k] * W'[k, n] ).
//
// Used for two rows of the hot path:
//  * the content projections Qc = X Wq, Kc = X Wk, V = X Wv (the write-up
//    takes these pixel content features as given; "Résumé technique" 2.A),
//    written in the head-padded layout [T][heads][DP] the attention kernel
//    loads with TMA (column n = head*DP + d maps to weight column head*dh + d
//    for d < dh and to a zero column otherwise);
//  * the CLA pointwise conv G = D Wpw + bpw followed by the sigmoid of the
//    gate (RIB/SST write-up section 2.3), written as bf16 [T][C].
//
// Both are HBM-bound (C/2 flop per byte with C <= 256), so the kernel is a
// persistent streaming design, one CTA per SM:
//  * W' is staged once per CTA, A tiles stream through two buffers, both in
//    the UMMA K-major 128-byte-swizzled layout: K split in atoms of 64
//    elements, each atom [rows][128 B] with the 16-byte chunks of row r
//    permuted by r % 8 (the TMA/UMMA swizzle);
//  * A tiles are loaded with 8-byte cp.async, one warp per row so every warp
//    instruction reads one contiguous channels-last row (rows of C bf16 are
//    only 8-byte aligned when C % 8 != 0, which rules out TMA tiles for A);
//    the next tile is in flight while this one runs;
//  * one thread issues the K/16 MMAs of a tile into a TMEM accumulator;
//  * the 128 threads drain TMEM (thread = token row) into a shared-memory
//    staging tile that one thread writes back asynchronously: TMA tensor
//    stores from a swizzled tile for the head-padded projection outputs
//    (conflict-free staging writes), one bulk copy of the contiguous [128][C]
//    rows for the gate.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "rib_internal.h"
#include "sm100.cuh"

namespace rib {

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 128;

struct GemmParams {
  const __nv_bfloat16* A;
  long long T;        // output rows (mode 0: B*Hp*Wp padded-image tokens)
  int B, H, W, Hp, Wp;
  int K, KP, mode, heads, dh, n_real, w_cols;
  int n_tiles;
  int box_n[3];       // mode 0: columns per TMA store box (64 -> 128B swizzle, 16 -> 32B swizzle)
  GemmJob jobs[3];
  int* err;
};


// K-major, 128-byte swizzle: element (row, k) of a [rows x KP] operand lives
// in K-atom k/64 at row*128 + ((k%64/8) ^ (row%8))*16 + (k%8)*2.
__device__ __forceinline__ uint32_t sw128_off(int row, int k, int rows) {
  return static_cast<uint32_t>((k >> 6) * rows * 128 + row * 128 + ((((k & 63) >> 3) ^ (row & 7)) << 4) + (k & 7) * 2);
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(src)), "r"(c0), "r"(c1) : "memory");
}
__device__ __forceinline__ void bulk_store(void* gdst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               ::"l"(reinterpret_cast<uint64_t>(gdst)), "r"(smem_u32(src)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ float sigmoid_fast(float v) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * v));
  return fmaf(0.5f, t, 0.5f);
}

__global__ void __launch_bounds__(kThreads, 1)
rib_token_gemm_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                      const __grid_constant__ CUtensorMap tm2, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int KP = p.KP;
  // this CTA's job, selected without dynamic indexing (which would put the
  // whole struct in local memory and reload it per element)
  const GemmJob job = blockIdx.y == 0 ? p.jobs[0] : (blockIdx.y == 1 ? p.jobs[1] : p.jobs[2]);
  const int N = job.N;
  const int box_n = blockIdx.y == 0 ? p.box_n[0] : (blockIdx.y == 1 ? p.box_n[1] : p.box_n[2]);
  const CUtensorMap* tmap = blockIdx.y == 0 ? &tm0 : (blockIdx.y == 1 ? &tm1 : &tm2);
  const int a_bytes = kTile * KP * 2;
  const int w_bytes = N * KP * 2;
  const int out_cols = p.mode == 0 ? N : p.n_real;
  const int o_bytes = (kTile * out_cols * 2 + 1023) & ~1023;
  uint8_t* sW = smem;
  uint8_t* sA[2] = {smem + w_bytes, smem + w_bytes + a_bytes};
  uint8_t* sO = smem + w_bytes + 2 * a_bytes;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sO + o_bytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar + 1);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(tmem_holder + 1);

  __shared__ float s_bias[256];
  for (int i = tid; i < 256; i += kThreads) s_bias[i] = (job.bias && i < p.n_real) ? job.bias[i] : 0.f;
  if (tid == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
    if (p.mode == 0) tma_prefetch_desc(tmap);
  }
  if (tid < 32) {
    tmem_alloc(tmem_holder, 256);
    tmem_relinquish();
  }
  // zero W' and both A buffers (K padding and the zero columns stay zero)
  for (int i = tid; i < (w_bytes + 2 * a_bytes) / 16; i += kThreads)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  // stage W': thread c copies weight column c (2-byte loads, coalesced across
  // threads) into row n of the K-major operand (n = c in mode 1, the
  // head-padded column in mode 0)
  {
    const uint16_t* Wt = static_cast<const uint16_t*>(job.Wt);
    for (int c = tid; c < p.w_cols; c += kThreads) {
      const int n = p.mode == 0 ? (c / p.dh) * job.DP + (c % p.dh) : c;
      if (n >= N) continue;
      for (int k0 = 0; k0 < p.K; k0 += 8) {
        uint16_t v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = (k0 + e < p.K) ? __ldg(Wt + static_cast<size_t>(k0 + e) * p.w_cols + c) : 0;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (k0 + e < p.K) *reinterpret_cast<uint16_t*>(sW + sw128_off(n, k0 + e, N)) = v[e];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, p.err};

  const int kq = p.K / 4;   // 8-byte chunks per A row
  // Thread tid owns row tid of every A tile (kTile == kThreads). Its source
  // row: mode 0 maps the padded-image token to the unpadded map (-1 in the
  // padding, which stays zero in the tile); mode 1 is the identity.
  // source row (in A) of output row t; -1 for padded-image tokens (mode 0)
  auto src_row = [&](long long t) -> long long {
    if (t >= p.T) return -2;
    if (p.mode != 0) return t;
    const int hw = p.Hp * p.Wp;
    const int b = static_cast<int>(t / hw);
    const int rem = static_cast<int>(t - static_cast<long long>(b) * hw);
    const int y = rem / p.Wp, x = rem - y * p.Wp;
    if (y >= p.H || x >= p.W) return -1;
    return (static_cast<long long>(b) * p.H + y) * p.W + x;
  };
  __shared__ long long s_src[2][kTile];   // per buffer: source row of each tile row
  const int warp = tid >> 5, lane = tid & 31;
  // Each thread maps one row, then each warp copies whole rows (8-byte
  // cp.async, lanes along the channels: one contiguous row per instruction).
  auto prefetch = [&](int tile, int buf) {
    const long long t0 = static_cast<long long>(tile) * kTile;
    s_src[buf][tid] = src_row(t0 + tid);
    __syncwarp();
    // rows r = 32*warp + i are mapped by lanes of this same warp
    for (int i = 0; i < 32; ++i) {
      const int r = warp * 32 + i;
      const long long sr = s_src[buf][r];
      if (sr == -2) break;
      uint8_t* rowp = sA[buf] + r * 128;
      for (int q = lane; q < kq; q += 32) {
        // chunk q = columns 4q..4q+3: atom q/16, 16-byte chunk (q%16)/2, half q%2
        uint8_t* dst = rowp + (q >> 4) * (kTile * 128) + ((((q & 15) >> 1) ^ (r & 7)) << 4) + (q & 1) * 8;
        if (sr >= 0) cp_async_8(dst, p.A + sr * p.K + q * 4);
        else *reinterpret_cast<uint2*>(dst) = make_uint2(0u, 0u);
      }
    }
  };

  const uint32_t idesc = idesc_bf16(128, N, false, false);
  const int row = tid;
  const uint32_t lane_off = static_cast<uint32_t>((tid / 32) * 32) << 16;

  int it = 0;
  int tile = blockIdx.x;
  if (tile < p.n_tiles) prefetch(tile, 0);
  cp_async_commit();
  for (; tile < p.n_tiles; tile += gridDim.x, ++it) {
    const int buf = it & 1;
    const int next = tile + gridDim.x;
    if (next < p.n_tiles) prefetch(next, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t a0 = smem_u32(sA[buf]), w0 = smem_u32(sW);
      for (int ks = 0; ks < KP / 16; ++ks) {
        // K step ks: atom ks/4, 32-byte offset (ks%4) inside the 128-byte row
        const uint32_t ka = (ks >> 2) * (kTile * 128) + (ks & 3) * 32;
        const uint32_t kw = (ks >> 2) * (N * 128) + (ks & 3) * 32;
        umma_ss(tmem, make_sdesc(a0 + ka, 16, 1024, SW_128B), make_sdesc(w0 + kw, 16, 1024, SW_128B), idesc,
                ks > 0 ? 1u : 0u);
      }
      umma_commit(bar);
      // the staging tile is rewritten below: the previous store must have read it
      bulk_wait_read0();
    }
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, it & 1, wc, 201));
    tc_fence_after();
    __syncthreads();   // staging free (thread 0 waited for the previous store's reads)
    const long long t0 = static_cast<long long>(tile) * kTile;
    if (ok) {
      for (int c0 = 0; c0 < N; c0 += 64) {
        uint32_t v[64];
        const int nb = (N - c0) >= 64 ? 4 : (N - c0) / 16;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q < nb) tmem_ld16(tmem + lane_off + c0 + 16 * q, *reinterpret_cast<uint32_t(*)[16]>(&v[16 * q]));
        tmem_wait_ld();
        if (p.mode == 0) {
          const float s = job.scale;
#pragma unroll
          for (int q = 0; q < 8; ++q) {      // 8 chunks of 8 columns
            const int c = c0 + 8 * q;
            if (c < N) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                f[e] = __uint_as_float(v[8 * q + e]) * s;
                if (((c + e) & (job.DP - 1)) == job.ones_col) f[e] = 1.f;
              }
              uint4 o;
              if (job.out_f16) {
                o = make_uint4(pack_f16x2(f[0], f[1]), pack_f16x2(f[2], f[3]), pack_f16x2(f[4], f[5]),
                               pack_f16x2(f[6], f[7]));
              } else {
                o = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                               pack_bf16x2(f[6], f[7]));
              }
              // box b holds columns [b*box_n, (b+1)*box_n) as rows of box_n*2
              // bytes; TMA swizzle: 16-byte chunk index XOR (row % 8) for
              // 128-byte rows, XOR ((row / 4) % 2) for 32-byte rows
              const int bx = c / box_n, cc = (c % box_n) / 8;
              uint32_t off;
              if (box_n == 64) off = bx * (kTile * 128) + row * 128 + ((cc ^ (row & 7)) << 4);
              else off = bx * (kTile * 32) + row * 32 + ((cc ^ ((row >> 2) & 1)) << 4);
              *reinterpret_cast<uint4*>(sO + off) = o;
            }
          }
        } else {
#pragma unroll
          for (int q = 0; q < 16; ++q) {     // 16 chunks of 4 columns
            const int c = c0 + 4 * q;
            if (c < p.n_real) {
              float g[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                g[e] = sigmoid_fast(__uint_as_float(v[4 * q + e]) + s_bias[c + e]);
              *reinterpret_cast<uint2*>(sO + (row * p.n_real + c) * 2) =
                  make_uint2(pack_bf16x2(g[0], g[1]), pack_bf16x2(g[2], g[3]));
            }
          }
        }
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    if (__syncthreads_or(ok ? 0 : 1)) break;   // also frees TMEM / the A buffer for the next tile
    const long long rows = (p.T - t0) < kTile ? (p.T - t0) : kTile;
    if (tid == 0) {
      if (p.mode == 0) {
        for (int bx = 0; bx < N / box_n; ++bx)
          tma_store_2d(tmap, sO + bx * kTile * box_n * 2, bx * box_n, static_cast<int>(t0));
      } else if ((rows * p.n_real * 2) % 16 == 0) {
        bulk_store(static_cast<__nv_bfloat16*>(job.out) + t0 * p.n_real, sO, static_cast<uint32_t>(rows * p.n_real * 2));
      }
      bulk_commit();
    }
    if (p.mode != 0 && (rows * p.n_real * 2) % 16 != 0 && row < rows) {
      // ragged last tile whose byte count is not a multiple of 16: plain stores
      const uint2* src = reinterpret_cast<const uint2*>(sO + row * p.n_real * 2);
      uint2* dst = reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(job.out) + (t0 + row) * p.n_real);
      for (int q = 0; q < p.n_real / 4; ++q) dst[q] = src[q];
    }
  }
  cp_async_wait<0>();
  if (tid == 0) bulk_wait0();
  tc_fence_before();
  __syncthreads();
  if (tid < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

cudaError_t launch_token_gemm(const GemmLaunch& g, cudaStream_t stream) {
  GemmParams p;
  p.A = static_cast<const __nv_bfloat16*>(g.A);
  p.B = g.B;
  p.H = g.H;
  p.W = g.W;
  p.Hp = g.mode == 0 ? g.Hp : g.H;
  p.Wp = g.mode == 0 ? g.Wp : g.W;
  p.T = static_cast<long long>(g.B) * p.Hp * p.Wp;
  p.K = g.K;
  p.KP = (g.K + 63) / 64 * 64;   // whole 128-byte swizzle atoms along K
  p.mode = g.mode;
  p.heads = g.heads;
  p.dh = g.dh;
  p.n_real = g.n_real;
  p.w_cols = g.w_cols;
  p.n_tiles = static_cast<int>((p.T + kTile - 1) / kTile);
  int n_max = 16, o_max = 0;
  for (int i = 0; i < 3; ++i) {
    p.jobs[i] = g.jobs[i];
    p.box_n[i] = (g.jobs[i].N % 64 == 0) ? 64 : 16;
    if (i < g.njobs) {
      n_max = g.jobs[i].N > n_max ? g.jobs[i].N : n_max;
      const int oc = g.mode == 0 ? g.jobs[i].N : g.n_real;
      o_max = oc > o_max ? oc : o_max;
    }
  }
  p.err = device_error_word();
  if (p.n_tiles == 0) return cudaSuccess;
  CUtensorMap maps[3];
  std::memset(maps, 0, sizeof(maps));
  if (g.mode == 0) {
    for (int j = 0; j < g.njobs; ++j) {
      const uint64_t dims[2] = {uint64_t(g.jobs[j].N), uint64_t(p.T)};
      const uint64_t strides[1] = {uint64_t(g.jobs[j].N) * 2};
      const uint32_t box[2] = {uint32_t(p.box_n[j]), uint32_t(kTile)};
      if (encode_tiled(&maps[j], g.jobs[j].out_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                       g.jobs[j].out, dims, strides, box,
                       p.box_n[j] == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
  }
  const size_t o_bytes = (static_cast<size_t>(kTile) * o_max * 2 + 1023) & ~size_t(1023);
  const size_t smem = static_cast<size_t>(n_max) * p.KP * 2 + 2 * kTile * p.KP * 2 + o_bytes + 64 + 1024;
  cudaError_t e = cudaFuncSetAttribute(rib_token_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // one CTA per SM (shared memory holds W' plus two A tiles and the staging
  // tile): all CTAs of the persistent grid must be co-resident or the last
  // ones run as a second wave
  const int sms = sm_count();
  int gx = sms / g.njobs;
  if (gx < 1) gx = 1;
  if (gx > p.n_tiles) gx = p.n_tiles;
  dim3 grid(gx, g.njobs);
  rib_token_gemm_kernel<<<grid, kThreads, smem, stream>>>(maps[0], maps[1], maps[2], p);
  return cudaGetLastError();
}

}  // namespace rib
