// Backward of the windowed RIB attention for sm_100a.
//
// For one window and head with S = Qc Kc^T + Qp Kp^T (Qc, Qp as stored: Qc
// carries 1/sqrt(dh), the cached Qp carries 1/sqrt(R)), z = s*S, P = softmax(z)
// and O = P V, the gradients from dO are
//   D   = rowsum(dO * O)
//   dS  = s * P * (dO V^T - D)          (gradient of S)
//   dQc = dS Kc,  dQp = dS Kp,  dKc = dS^T Qc,  dKp = dS^T Qp,  dV = P^T dO
// i.e. dQ = dS K split at the content/position boundary of the concatenated
// K = [Kc, Kp] (RIB/SST write-up, section 2.2: one product of the
// concatenations), and dQp/dKp summed over every window and image feed the
// coordinate MLP (rib_pos_encode_bwd).
//
// The per-row constants live inside the tensor-core products, so the
// elementwise work per score is one exponential and one multiply:
//  * rib_attention_bwd_prep stores dO'' = s * dO with -s*D, split into a bf16
//    pair (hi, lo), in columns dh and dh+1; V's columns d >= dh are 1, so
//    dP'' = dO'' V^T = s * (dO V^T - D) and dS = P * dP''.
//  * For padded heads (dh + 2 <= DP) the first step of the backward writes
//    Q'' = [bf16(l2 * Qc) with -log2(e) * lse split into (hi, lo) in columns
//    dh, dh+1, bf16(l2 * Qp)] per token (l2 = s * log2(e)); Kc's columns d >=
//    dh are 1, so Q'' K^T = l2 * S - log2(e) * lse and P = 2^(Q'' K^T) needs no
//    lse at all.
//    The products with Q'' as an operand carry the factor l2 (dKc, dKp) and
//    those with dO'' the factor s (dV); the epilogues divide it out.
//  * Otherwise (dh == DP) P = 2^(l2 * S - log2(e) * lse) from the forward's lse.
//
// Two kernels:
//  * dq kernel, one 128-query tile per CTA, streaming 64-key tiles:
//    S and dP'' by tcgen05 into TMEM (one buffer each), the elementwise
//    warpgroup forms dS (bf16, two TMEM buffers), and [dQc | dQp] accumulates
//    in TMEM as one product per K step: dS (A operand from TMEM) times the
//    key tile's [Kc | Kp] (N = DP + 16).
//  * dkv kernel, one 128-key tile per CTA, streaming 64-query tiles: S^T and
//    dP''^T (keys in TMEM lanes); the elementwise warps read both, which
//    frees them for the next tile's products, and write P^T and dS^T (bf16)
//    to shared memory; dV += P^T dO'' and [dKc | dKp] += dS^T [Qc'' | Qp'']
//    accumulate in TMEM. The next tile's S^T and dP''^T thus run on the
//    tensor cores while the current tile's exponentials run.
//  The streamed tile's content and position features (Kc, Kp in dq; Qc'',
//  Qp'' in dkv) arrive without swizzle as 8-feature atoms (1 KB each: 64
//  rows of 8 features, 16 bytes a row), so the same bytes serve as the K-major
//  operand of the score product and as the MN-major operand of the merged
//  gradient product, whose N runs over both feature groups.
// Both kernels hold 256 TMEM columns, so two CTAs share an SM.
// Warp roles: warp 0 TMA producer; warps 1 and 6 one MMA-issuing thread each
// (warp 1 also owns TMEM): one thread issues an M = 128, K = 16 product
// about every 55 cycles at N <= 64 while the SM retires one every ~40-48,
// and each stream waits on its own dependencies, so the score products (S,
// dP'') and the accumulating products go out from different threads; warps 2-5 one elementwise warpgroup (thread =
// TMEM lane = query row or key row), which reads the score tiles in two
// halves and releases them after the second load. POLY of every 8
// exponential pairs run on the FMA pipe.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "rib_internal.h"
#include "sm100.cuh"

namespace rib {

namespace {

constexpr int kR = 16;
constexpr int kBwdThreads = 224;   // 7 warps: producer, two MMA issuers, four elementwise
constexpr float kLog2e = 1.4426950408889634f;

enum BwdSite : int {
  SITE_B_Q = 301, SITE_B_KV_FULL = 302, SITE_B_KV_EMPTY = 303, SITE_B_S_FREE = 304, SITE_B_DS_FULL = 305,
  SITE_B_S_FULL = 306, SITE_B_DQ_DONE = 307, SITE_B_DONE = 308, SITE_B_DRAIN = 309,
};

__device__ __forceinline__ bool warp_all_b(bool v) { return __all_sync(0xffffffffu, v); }

struct BwdParams {
  int B, heads, dh, M, Hp, Wp, nwx, nwy;
  int tc, tr, tiles_x;      // 128-token tiles of the CTA's own side
  int tc2, tr2, tiles_x2;   // 64-token tiles of the streamed side
  int n_stream;             // streamed 64-token tiles per window
  int n_own;                // 128-token tiles per window
  float scale_log2, scale;
  float inv_scale, inv_scale_log2;   // epilogue factors of dV and (folded) dKc, dKp
  const float* lse;         // [B][heads][Hp][Wp]
  float* out_c;             // dq: dQc, dkv: dKc   fp32 [B][Hp][Wp][heads][32]
  float* out_v;             // dkv: dV            fp32 [B][Hp][Wp][heads][32]
  float* out_p;             // partials fp32 [B*nW][heads][M*M][16]
  int* err;
};

// dq kernel (two CTAs per SM, 256 columns each): one S and one dP buffer at
// 0 and 64 (the issuer starts S(j+1) once the elementwise warps have read
// S(j) and dP(j)), two dS buffers at 128 and 160, dQc at 192 (32), dQp at 224.
// dQ accumulates [dQc | dQp] at kDqA0 (DP + 16 columns)
constexpr uint32_t kDqS = 0, kDqDP = 64, kDqDS = 128, kDqA0 = 192, kDqCols = 256;
// dkv kernel (two CTAs per SM, 256 columns each): S^T at 0, dP^T at 64 (both
// free again once the elementwise warps have read them: P^T and dS^T go to
// shared memory); dV at 128, dKc at 160, dKp at 192.
// dK accumulates [dKc | dKp] at kDkvA1 (DP + 16 columns)
constexpr uint32_t kDkvS = 0, kDkvR = 64, kDkvA0 = 128, kDkvA1 = 160, kDkvCols = 256;

template <int DP>
struct BwdLay {
  // own-side tile (128 rows), loaded once
  static constexpr int OWN_C = 128 * DP * 2;
  static constexpr int OWN_P = 128 * kR * 2;
  static constexpr int OWN_V = 128 * 32 * 2;            // dq: dO, dkv: V (bf16)
  // streamed tile (64 rows) + per-row lse/D (dkv only)
  static constexpr int ST_C = 64 * DP * 2;
  static constexpr int ST_P = 64 * kR * 2;
  static constexpr int ST_V = 64 * 32 * 2;               // dq: V, dkv: dO (bf16)
  static constexpr int ST_LD = 64 * 4;                   // dkv without the fold: the tile's lse
  static constexpr int ST_RAW = ST_C + ST_P + ST_V + ST_LD;
  static constexpr int STAGE = (ST_RAW + 1023) / 1024 * 1024;
  static constexpr int NS = 4;
  static constexpr int OFF_OWN = 0;
  static constexpr int OFF_ST = OWN_C + OWN_P + OWN_V;
  // dkv: P^T and dS^T of the current query tile, [128 keys][64 queries] bf16
  // each, K-major with the 128-byte swizzle (the A operands of the
  // accumulating MMAs)
  static constexpr int OFF_PDS = OFF_ST + NS * STAGE;
  static constexpr int PDS_TILE = 128 * 64 * 2;
  static constexpr int OFF_BAR = OFF_PDS + 2 * PDS_TILE;
  // own_full, st_full[NS], st_empty[NS], s_full[2], s_free[2], x_full[2], x_done[2], done
  static constexpr int NBAR = 1 + 2 * NS + 8 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int ALLOC = OFF_MISC + 16 + 1024;
  static constexpr uint32_t SW_C = DP == 32 ? SW_64B : SW_32B;
  static constexpr uint32_t SBO_C = 8 * DP * 2;
};

__device__ __forceinline__ uint32_t pack_bf16x2_b(float lo, float hi) { return pack_bf16x2(lo, hi); }

// -------------------------------------------------------------------------
// dQ kernel
// -------------------------------------------------------------------------
template <int DP, bool FOLD, int POLY>
__global__ void __launch_bounds__(kBwdThreads, 2)
rib_attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qp,
                       const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_kp, const __grid_constant__ CUtensorMap tm_v,
                       const BwdParams p) {
  using Lay = BwdLay<DP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* own_full = bars;
  uint64_t* st_full = bars + 1;
  uint64_t* st_empty = bars + 1 + Lay::NS;
  uint64_t* s_full = bars + 1 + 2 * Lay::NS;   // single S/dP buffer: [0] used
  uint64_t* s_free = s_full + 2;
  uint64_t* x_full = s_full + 4;     // dS written
  uint64_t* x_done = s_full + 6;     // dQ MMAs of that buffer done
  uint64_t* done = s_full + 8;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + Lay::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int u = blockIdx.x;
  const int qt = u % p.n_own;
  u /= p.n_own;
  const int head = u % p.heads;
  const int w = u / p.heads;
  const int wx = w % p.nwx, wy = (w / p.nwx) % p.nwy, b = w / (p.nwx * p.nwy);
  const int y0 = wy * p.M, x0 = wx * p.M;
  const int n = p.n_stream;

  if (threadIdx.x == 0) {
    mbar_init(own_full, 1);
    for (int s = 0; s < Lay::NS; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 2);   // released by both issuers
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&x_full[i], 4);
      mbar_init(&x_done[i], 1);
    }
    mbar_init(done, 2);
    *abort_flag = 0u;
    tmem_holder[2] = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kDqCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, p.err};
  const WaitCtx drain{reinterpret_cast<volatile uint32_t*>(tmem_holder + 2), p.err};
  uint8_t* own = smem + Lay::OFF_OWN;

  if (warp == 0) {
    if (lane == 0) {
      const int ty = (qt / p.tiles_x) * p.tr, tx = (qt % p.tiles_x) * p.tc;
      mbar_arrive_expect_tx(own_full, Lay::OWN_C + Lay::OWN_P + Lay::OWN_V);
      tma_load_5d(own, &tm_q, own_full, 0, head, x0 + tx, y0 + ty, b);
      if constexpr (FOLD) tma_load_5d(own + Lay::OWN_C, &tm_qp, own_full, 0, head, x0 + tx, y0 + ty, b);
      else tma_load_4d(own + Lay::OWN_C, &tm_qp, own_full, 0, tx, ty, head);
      tma_load_5d(own + Lay::OWN_C + Lay::OWN_P, &tm_do, own_full, 0, head, x0 + tx, y0 + ty, b);
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % Lay::NS;
        if (i >= Lay::NS && !mbar_wait(&st_empty[st], ((i / Lay::NS) - 1) & 1, wc, SITE_B_KV_EMPTY)) break;
        uint8_t* sb = smem + Lay::OFF_ST + st * Lay::STAGE;
        const int ky = (i / p.tiles_x2) * p.tr2, kx = (i % p.tiles_x2) * p.tc2;
        mbar_arrive_expect_tx(&st_full[st], Lay::ST_C + Lay::ST_P + Lay::ST_V);
        // Kc, Kp as unswizzled 1 KB atoms of 8 features x 64 keys: one tile
        // that is both the K-major B operand of S and the MN-major B operand
        // of the merged dQ product
#pragma unroll
        for (int a = 0; a < DP / 8; ++a) tma_load_5d(sb + a * 1024, &tm_k, &st_full[st], 8 * a, head, x0 + kx, y0 + ky, b);
#pragma unroll
        for (int a = 0; a < kR / 8; ++a) tma_load_4d(sb + Lay::ST_C + a * 1024, &tm_kp, &st_full[st], 8 * a, kx, ky, head);
        tma_load_5d(sb + Lay::ST_C + Lay::ST_P, &tm_v, &st_full[st], 0, head, x0 + kx, y0 + ky, b);
        issued = i + 1;
      }
      mbar_wait(own_full, 0, drain, SITE_B_DRAIN);
      for (int i = issued - Lay::NS > 0 ? issued - Lay::NS : 0; i < issued; ++i)
        mbar_wait(&st_full[i % Lay::NS], (i / Lay::NS) & 1, drain, SITE_B_DRAIN);
    }
  } else if (warp == 1 || warp == 6) {
    // two MMA issuers with their own instruction streams: warp 1 issues S and
    // dP'', warp 6 the dQc and dQp products
    if (lane == 0) {
      const bool first = warp == 1;
      constexpr uint32_t id_s = idesc_bf16(128, 64, false, false);
      constexpr uint32_t id_dp = idesc_bf16(128, 64, false, false);
      constexpr uint32_t id_q = idesc_bf16(128, DP + kR, false, true);
      const uint32_t sq = smem_u32(own), sqp = sq + Lay::OWN_C, sdo = sqp + Lay::OWN_P;
      const uint32_t sst = smem_u32(smem + Lay::OFF_ST);
      auto issue_s = [&](int j) {
        const int st = j % Lay::NS;
        const uint32_t kb = sst + st * Lay::STAGE, kpb = kb + Lay::ST_C, vb = kpb + Lay::ST_P;
        const uint32_t dS = tmem + kDqS, dDP = tmem + kDqDP;
#pragma unroll
        for (int k = 0; k < DP / 16; ++k)
          umma_ss(dS, make_sdesc(sq + 32 * k, 16, Lay::SBO_C, Lay::SW_C), make_sdesc(kb + 2048 * k, 1024, 128, SW_NONE),
                  id_s, k > 0 ? 1u : 0u);
        umma_ss(dS, make_sdesc(sqp, 16, 256, SW_32B), make_sdesc(kpb, 1024, 128, SW_NONE), id_s, 1u);
#pragma unroll
        for (int k = 0; k < 2; ++k)
          umma_ss(dDP, make_sdesc(sdo + 32 * k, 16, 512, SW_64B), make_sdesc(vb + 32 * k, 16, 512, SW_64B), id_dp,
                  k > 0 ? 1u : 0u);
        umma_commit(s_full);
        umma_commit(&st_empty[st]);
      };
      auto issue_dq = [&](int j) {
        const int st = j % Lay::NS, bb = j & 1;
        const uint32_t kb = sst + st * Lay::STAGE, kpb = kb + Lay::ST_C;
        const uint32_t a = tmem + kDqDS + 32u * bb;
        // [dQc | dQp] += dS [Kc | Kp]: K MN-major without swizzle (LBO: 8-key
        // groups, 128 B; SBO: feature atoms, 1 KB), one product per K step
#pragma unroll
        for (int k = 0; k < 4; ++k)   // 64 keys = 4 K-steps of 16
          umma_ts(tmem + kDqA0, a + 8u * k, make_sdesc(kb + 256 * k, 128, 1024, SW_NONE), id_q, (j > 0 || k > 0) ? 1u : 0u);
        umma_commit(&x_done[bb]);
        umma_commit(&st_empty[st]);
      };
      bool ok = mbar_wait(own_full, 0, wc, SITE_B_Q);
      if (first) {
        for (int j = 0; ok && j < n; ++j) {
          if (!(ok = mbar_wait(&st_full[j % Lay::NS], (j / Lay::NS) & 1, wc, SITE_B_KV_FULL))) break;
          // single S/dP buffer: the elementwise warps have read S(j-1), dP(j-1)
          if (j >= 1 && !(ok = mbar_wait(s_free, (j - 1) & 1, wc, SITE_B_S_FREE))) break;
          tc_fence_after();
          issue_s(j);
        }
      } else {
        for (int j = 0; ok && j < n; ++j) {
          if (!(ok = mbar_wait(&x_full[j & 1], (j >> 1) & 1, wc, SITE_B_DS_FULL))) break;
          tc_fence_after();
          issue_dq(j);
        }
      }
      umma_commit(done);
      mbar_wait(done, 0, drain, SITE_B_DONE);
    }
  } else {
    // elementwise warpgroup: thread = query row
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int ty = (qt / p.tiles_x) * p.tr + row / p.tc, tx = (qt % p.tiles_x) * p.tc + row % p.tc;
    const int y = y0 + ty, x = x0 + tx;
    // without the fold: P = 2^(l2 S - l2 lse) with this row's lse
    const float lse2 = FOLD ? 0.f : __ldg(p.lse + ((static_cast<size_t>(b) * p.heads + head) * p.Hp + y) * p.Wp + x) * kLog2e;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int bb = j & 1;
      ok = warp_all_b(mbar_wait(s_full, j & 1, wc, SITE_B_S_FULL));
      if (!ok) break;
      if (j >= 2) {
        ok = warp_all_b(mbar_wait(&x_done[bb], ((j - 2) >> 1) & 1, wc, SITE_B_DQ_DONE));
        if (!ok) break;
      }
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {   // keys 32h .. 32h+31
        uint32_t sv[32], dv[32];
        tmem_ld32(tmem + lane_off + kDqS + 32u * h, sv);
        tmem_ld32(tmem + lane_off + kDqDP + 32u * h, dv);
        tmem_wait_ld();
        if (h == 1) {
          // S(j) and dP(j) are in registers: the next tile's products may overwrite them
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free);
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0 = __uint_as_float(sv[2 * i]), x1 = __uint_as_float(sv[2 * i + 1]);
          if constexpr (!FOLD) {
            x0 = fmaf(x0, sl2, -lse2);
            x1 = fmaf(x1, sl2, -lse2);
          }
          float p0, p1;
          if ((i & 7) < POLY) {
            exp2_poly_x2(x0, x1, p0, p1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          // dS = P * dP'' (dP'' = s (dO V^T - D) from the product)
          float d0, d1;
          f2_unpack(f2_mul(f2_pack(p0, p1), f2_pack(__uint_as_float(dv[2 * i]), __uint_as_float(dv[2 * i + 1]))), d0, d1);
          pk[i] = pack_bf16x2_b(d0, d1);
        }
        tmem_st16(tmem + lane_off + kDqDS + 32u * bb + 16u * h, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&x_full[bb]);
    }
    if (ok && n > 0) {
      ok = warp_all_b(mbar_wait(&x_done[(n - 1) & 1], ((n - 1) >> 1) & 1, wc, SITE_B_DQ_DONE));
      if (ok) {
        tc_fence_after();
        uint32_t qc[32], qp[16];
        tmem_ld32(tmem + lane_off + kDqA0, qc);
        tmem_ld16(tmem + lane_off + kDqA0 + DP, qp);   // the merged product's rank columns
        tmem_wait_ld();
        float4* oc = reinterpret_cast<float4*>(
            p.out_c + (((static_cast<size_t>(b) * p.Hp + y) * p.Wp + x) * p.heads + head) * 32);
#pragma unroll
        for (int d = 0; d < 32; d += 4)
          oc[d / 4] = (d < DP) ? make_float4(__uint_as_float(qc[d]), __uint_as_float(qc[d + 1]), __uint_as_float(qc[d + 2]),
                                             __uint_as_float(qc[d + 3]))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        const int t = ty * p.M + tx;
        float4* op = reinterpret_cast<float4*>(p.out_p + ((static_cast<size_t>(w) * p.heads + head) * p.M * p.M + t) * kR);
#pragma unroll
        for (int r = 0; r < kR; r += 4)
          op[r / 4] = make_float4(__uint_as_float(qp[r]), __uint_as_float(qp[r + 1]), __uint_as_float(qp[r + 2]),
                                  __uint_as_float(qp[r + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kDqCols);
  }
}

// -------------------------------------------------------------------------
// dK / dV kernel
// -------------------------------------------------------------------------
template <int DP, bool FOLD, int POLY>
__global__ void __launch_bounds__(kBwdThreads, 2)
rib_attn_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kp,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_qp, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_lse, const BwdParams p) {
  using Lay = BwdLay<DP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* own_full = bars;
  uint64_t* st_full = bars + 1;
  uint64_t* st_empty = bars + 1 + Lay::NS;
  uint64_t* s_full = bars + 1 + 2 * Lay::NS;   // S^T(i), dP^T(i) in TMEM (and every earlier MMA done)
  uint64_t* s_free = s_full + 2;                // S^T(i), dP^T(i) read by the elementwise warps
  uint64_t* x_full = s_full + 4;                // P^T(i) and dS^T(i) written to shared memory
  uint64_t* pds_free = s_full + 6;              // the accumulating MMAs of tile i have read them
  uint64_t* done = s_full + 8;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + Lay::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int u = blockIdx.x;
  const int kt = u % p.n_own;
  u /= p.n_own;
  const int head = u % p.heads;
  const int w = u / p.heads;
  const int wx = w % p.nwx, wy = (w / p.nwx) % p.nwy, b = w / (p.nwx * p.nwy);
  const int y0 = wy * p.M, x0 = wx * p.M;
  const int n = p.n_stream;

  if (threadIdx.x == 0) {
    mbar_init(own_full, 1);
    for (int s = 0; s < Lay::NS; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 2);   // released by both issuers
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(x_full, 4);
    mbar_init(pds_free, 1);   // the second issuer's accumulating MMAs
    mbar_init(done, 2);
    *abort_flag = 0u;
    tmem_holder[2] = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kDkvCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, p.err};
  const WaitCtx drain{reinterpret_cast<volatile uint32_t*>(tmem_holder + 2), p.err};
  uint8_t* own = smem + Lay::OFF_OWN;

  if (warp == 0) {
    if (lane == 0) {
      const int ty = (kt / p.tiles_x) * p.tr, tx = (kt % p.tiles_x) * p.tc;
      mbar_arrive_expect_tx(own_full, Lay::OWN_C + Lay::OWN_P + Lay::OWN_V);
      tma_load_5d(own, &tm_k, own_full, 0, head, x0 + tx, y0 + ty, b);
      tma_load_4d(own + Lay::OWN_C, &tm_kp, own_full, 0, tx, ty, head);
      tma_load_5d(own + Lay::OWN_C + Lay::OWN_P, &tm_v, own_full, 0, head, x0 + tx, y0 + ty, b);
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % Lay::NS;
        if (i >= Lay::NS && !mbar_wait(&st_empty[st], ((i / Lay::NS) - 1) & 1, wc, SITE_B_KV_EMPTY)) break;
        uint8_t* sb = smem + Lay::OFF_ST + st * Lay::STAGE;
        const int qy = (i / p.tiles_x2) * p.tr2, qx = (i % p.tiles_x2) * p.tc2;
        mbar_arrive_expect_tx(&st_full[st], Lay::ST_C + Lay::ST_P + Lay::ST_V + (FOLD ? 0 : Lay::ST_LD));
        // Q'' as unswizzled 1 KB atoms of 8 features x 64 queries (content
        // atoms, then the two rank atoms): one tile that is both the K-major
        // B operand of S^T and the MN-major B operand of the merged dK product
#pragma unroll
        for (int a = 0; a < DP / 8; ++a) tma_load_5d(sb + a * 1024, &tm_q, &st_full[st], 8 * a, head, x0 + qx, y0 + qy, b);
#pragma unroll
        for (int a = 0; a < kR / 8; ++a) {
          if constexpr (FOLD) tma_load_5d(sb + Lay::ST_C + a * 1024, &tm_qp, &st_full[st], 8 * a, head, x0 + qx, y0 + qy, b);
          else tma_load_4d(sb + Lay::ST_C + a * 1024, &tm_qp, &st_full[st], 8 * a, qx, qy, head);
        }
        tma_load_5d(sb + Lay::ST_C + Lay::ST_P, &tm_do, &st_full[st], 0, head, x0 + qx, y0 + qy, b);
        if constexpr (!FOLD)
          tma_load_4d(sb + Lay::ST_C + Lay::ST_P + Lay::ST_V, &tm_lse, &st_full[st], x0 + qx, y0 + qy, head, b);
        issued = i + 1;
      }
      mbar_wait(own_full, 0, drain, SITE_B_DRAIN);
      for (int i = issued - Lay::NS > 0 ? issued - Lay::NS : 0; i < issued; ++i)
        mbar_wait(&st_full[i % Lay::NS], (i / Lay::NS) & 1, drain, SITE_B_DRAIN);
    }
  } else if (warp == 1 || warp == 6) {
    // two MMA issuers, each with its own instruction stream (a thread's
    // tcgen05.mma stream runs one instruction at a time; two streams
    // overlap): warp 1 issues S^T and dP''^T (5 per tile), warp 6 dV and the
    // merged [dKc | dKp] (8 per tile: dK over the N = DP + 16 features of the
    // unswizzled Q'' tile is one product per K step)
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16(128, 64, false, false);
      constexpr uint32_t id_dp = idesc_bf16(128, 64, false, false);
      constexpr uint32_t id_v = idesc_bf16(128, 32, false, true);
      constexpr uint32_t id_k = idesc_bf16(128, DP + kR, false, true);
      const bool first = warp == 1;
      const uint32_t sk = smem_u32(own), skp = sk + Lay::OWN_C, sv = skp + Lay::OWN_P;
      const uint32_t sst = smem_u32(smem + Lay::OFF_ST);
      auto issue_s = [&](int i) {
        const int st = i % Lay::NS;
        const uint32_t qb = sst + st * Lay::STAGE, qpb = qb + Lay::ST_C, dob = qpb + Lay::ST_P;
        const uint32_t dS = tmem + kDkvS, dDP = tmem + kDkvR;
        // Q'' K-major without swizzle: 16 features = two atoms (LBO 1 KB), 8-query groups 128 B apart (SBO)
#pragma unroll
        for (int k = 0; k < DP / 16; ++k)
          umma_ss(dS, make_sdesc(sk + 32 * k, 16, Lay::SBO_C, Lay::SW_C), make_sdesc(qb + 2048 * k, 1024, 128, SW_NONE),
                  id_s, k > 0 ? 1u : 0u);
        umma_ss(dS, make_sdesc(skp, 16, 256, SW_32B), make_sdesc(qpb, 1024, 128, SW_NONE), id_s, 1u);
#pragma unroll
        for (int k = 0; k < 2; ++k)
          umma_ss(dDP, make_sdesc(sv + 32 * k, 16, 512, SW_64B), make_sdesc(dob + 32 * k, 16, 512, SW_64B), id_dp,
                  k > 0 ? 1u : 0u);
        umma_commit(s_full);
        umma_commit(&st_empty[st]);   // this issuer's reads of the stage (Q'', dO'')
      };
      const uint32_t spds = smem_u32(smem + Lay::OFF_PDS);
      // the accumulating MMAs of tile i (second issuer): dV += P^T dO'' and
      // [dKc | dKp] += dS^T [Qc'' | Qp''] (Q'' MN-major without swizzle: 8
      // features per atom; in this layout the descriptor takes the K-direction
      // stride (8-query groups, 128 B) as LBO and the MN-direction stride
      // (feature atoms, 1 KB) as SBO)
      auto issue_acc = [&](int i) {
        const int st = i % Lay::NS;
        const uint32_t qb = sst + st * Lay::STAGE, qpb = qb + Lay::ST_C, dob = qpb + Lay::ST_P;
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // 64 queries = 4 K-steps of 16 (32 bytes of the 128-byte rows)
          const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
          const uint64_t aP = make_sdesc(spds + 32 * k, 16, 1024, SW_128B);
          umma_ss(tmem + kDkvA0, aP, make_sdesc(dob + k * 16 * 64, 8192, 512, SW_64B), id_v, acc);
          const uint64_t aS = make_sdesc(spds + Lay::PDS_TILE + 32 * k, 16, 1024, SW_128B);
          umma_ss(tmem + kDkvA1, aS, make_sdesc(qb + 256 * k, 128, 1024, SW_NONE), id_k, acc);
        }
        umma_commit(pds_free);
        umma_commit(&st_empty[st]);
      };
      // First issuer: S^T(i), dP^T(i) go out as soon as the elementwise warps
      // have read tile i-1's (s_free), so they run while tile i-1's
      // exponentials do. Second issuer: dV and dK of each tile once its P^T
      // and dS^T are in shared memory (x_full).
      bool ok = mbar_wait(own_full, 0, wc, SITE_B_Q);
      if (first) {
        for (int i = 0; ok && i < n; ++i) {
          if (!(ok = mbar_wait(&st_full[i % Lay::NS], (i / Lay::NS) & 1, wc, SITE_B_KV_FULL))) break;
          if (i >= 1 && !(ok = mbar_wait(s_free, (i - 1) & 1, wc, SITE_B_S_FREE))) break;
          tc_fence_after();
          issue_s(i);
        }
      } else {
        for (int i = 0; ok && i < n; ++i) {
          if (!(ok = mbar_wait(x_full, i & 1, wc, SITE_B_DS_FULL))) break;
          tc_fence_after();
          issue_acc(i);
        }
      }
      umma_commit(done);
      mbar_wait(done, 0, drain, SITE_B_DONE);
    }
  } else {
    // elementwise warpgroup: thread = key row; columns = the 64 queries of the tile
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      ok = warp_all_b(mbar_wait(s_full, i & 1, wc, SITE_B_S_FULL));
      if (!ok) break;
      tc_fence_after();
      const float* ld = nullptr;
      if constexpr (!FOLD) {
        // the tile's lse was written by TMA into the stage: order the reads
        // after the stage's own barrier (complete by now; the stage is not
        // refilled before this step's accumulate MMAs have run)
        ok = warp_all_b(mbar_wait(&st_full[i % Lay::NS], (i / Lay::NS) & 1, wc, SITE_B_KV_FULL));
        if (!ok) break;
        ld = reinterpret_cast<const float*>(smem + Lay::OFF_ST + (i % Lay::NS) * Lay::STAGE + Lay::ST_C + Lay::ST_P +
                                            Lay::ST_V);
      }
      uint8_t* prow = smem + Lay::OFF_PDS + row * 128;   // this key's row of P^T (dS^T one tile further)
#pragma unroll
      for (int h = 0; h < 2; ++h) {   // queries 32h .. 32h+31
        uint32_t sv[32], dv[32];
        tmem_ld32(tmem + lane_off + kDkvS + 32u * h, sv);
        tmem_ld32(tmem + lane_off + kDkvR + 32u * h, dv);
        tmem_wait_ld();
        if (h == 1) {
          // S^T(i) and dP''^T(i) are in registers: the next tile's products may overwrite them
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free);
        }
        uint32_t pp[16], ds[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int q = 32 * h + 2 * c;
          float x0 = __uint_as_float(sv[2 * c]), x1 = __uint_as_float(sv[2 * c + 1]);
          if constexpr (!FOLD) {
            x0 = fmaf(x0, sl2, -ld[q] * kLog2e);
            x1 = fmaf(x1, sl2, -ld[q + 1] * kLog2e);
          }
          float p0, p1;
          if ((c & 7) < POLY) {
            exp2_poly_x2(x0, x1, p0, p1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          // dS^T = P^T * dP''^T
          float d0, d1;
          f2_unpack(f2_mul(f2_pack(p0, p1), f2_pack(__uint_as_float(dv[2 * c]), __uint_as_float(dv[2 * c + 1]))), d0,
                    d1);
          pp[c] = pack_bf16x2(p0, p1);
          ds[c] = pack_bf16x2_b(d0, d1);
        }
        if (h == 0 && i >= 1) {
          // the accumulating MMAs of the previous tile have read P^T and dS^T
          ok = warp_all_b(mbar_wait(pds_free, (i - 1) & 1, wc, SITE_B_DQ_DONE));
          if (!ok) break;
        }
        // queries 32h .. 32h+31 = 16-byte chunks 4h .. 4h+3 of the row, permuted by row % 8
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int off = (((4 * h + c) ^ (row & 7)) << 4);
          *reinterpret_cast<uint4*>(prow + off) = make_uint4(pp[4 * c], pp[4 * c + 1], pp[4 * c + 2], pp[4 * c + 3]);
          *reinterpret_cast<uint4*>(prow + Lay::PDS_TILE + off) =
              make_uint4(ds[4 * c], ds[4 * c + 1], ds[4 * c + 2], ds[4 * c + 3]);
        }
      }
      if (!ok) break;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(x_full);
    }
    if (ok && n > 0) {
      ok = warp_all_b(mbar_wait(done, 0, wc, SITE_B_DQ_DONE));
      if (ok) {
        tc_fence_after();
        uint32_t vv[32], kc[32], kp[16];
        tmem_ld32(tmem + lane_off + kDkvA0, vv);
        tmem_ld32(tmem + lane_off + kDkvA1, kc);
        tmem_ld16(tmem + lane_off + kDkvA1 + DP, kp);   // the merged product's rank columns
        tmem_wait_ld();
        const int ty = (kt / p.tiles_x) * p.tr + row / p.tc, tx = (kt % p.tiles_x) * p.tc + row % p.tc;
        const int y = y0 + ty, x = x0 + tx;
        const size_t base = (((static_cast<size_t>(b) * p.Hp + y) * p.Wp + x) * p.heads + head) * 32;
        float4* ov = reinterpret_cast<float4*>(p.out_v + base);
        float4* ok4 = reinterpret_cast<float4*>(p.out_c + base);
        // dV came from dO'' = s dO; with the fold, dKc and dKp from Q'' = l2 Q
        const float fv = p.inv_scale, fk = FOLD ? p.inv_scale_log2 : 1.f;
#pragma unroll
        for (int d = 0; d < 32; d += 4) {
          ov[d / 4] = make_float4(__uint_as_float(vv[d]) * fv, __uint_as_float(vv[d + 1]) * fv,
                                  __uint_as_float(vv[d + 2]) * fv, __uint_as_float(vv[d + 3]) * fv);
          ok4[d / 4] = (d < DP) ? make_float4(__uint_as_float(kc[d]) * fk, __uint_as_float(kc[d + 1]) * fk,
                                              __uint_as_float(kc[d + 2]) * fk, __uint_as_float(kc[d + 3]) * fk)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const int t = ty * p.M + tx;
        float4* op = reinterpret_cast<float4*>(p.out_p + ((static_cast<size_t>(w) * p.heads + head) * p.M * p.M + t) * kR);
#pragma unroll
        for (int r = 0; r < kR; r += 4)
          op[r / 4] = make_float4(__uint_as_float(kp[r]) * fk, __uint_as_float(kp[r + 1]) * fk,
                                  __uint_as_float(kp[r + 2]) * fk, __uint_as_float(kp[r + 3]) * fk);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kDkvCols);
  }
}

// -------------------------------------------------------------------------
// elementwise helpers
// -------------------------------------------------------------------------
// dO'' = s * dY * gate in the padded bf16 layout with -s*D as a bf16 (hi, lo)
// pair in columns dh and dh+1 and zeros past them (all zero in the padding),
// D = rowsum(dO * O) from the stored bf16 values (Dsum holds it unscaled),
// dG = dY * O * gate * (1 - gate) (optional).
__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ dY, const __nv_bfloat16* __restrict__ gate,
                                const __nv_bfloat16* __restrict__ O, __nv_bfloat16* __restrict__ dO, float* __restrict__ Dsum,
                                __nv_bfloat16* __restrict__ dG, int B, int H, int W, int C, int heads, int Hp, int Wp,
                                float sc) {
  // four threads per (padded token, head), eight output columns each; the
  // four are consecutive lanes, so D is summed over them by shuffles
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long total = static_cast<long long>(B) * Hp * Wp * heads;
  const long long th = gid >> 2;
  const int g = static_cast<int>(gid & 3);
  const bool in_range = th < total;
  const int head = static_cast<int>(th % heads);
  const long long pix = th / heads;
  const int xp = static_cast<int>(pix % Wp);
  const int yp = static_cast<int>((pix / Wp) % Hp);
  const int b = static_cast<int>(pix / (static_cast<long long>(Wp) * Hp));
  const int dh = C / heads;
  const int DP = (dh + 15) / 16 * 16;
  const bool real = in_range && yp < H && xp < W;
  const int d0 = 8 * g;
  float v[8], o[8];
  float dsum = 0.f;   // sum of the stored dO'' times O: s * D
  size_t cb = 0;
  uint32_t dyw[4] = {0u, 0u, 0u, 0u}, gw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = o[e] = 0.f;
  if (real && d0 < dh) {
    cb = ((static_cast<size_t>(b) * H + yp) * W + xp) * C + static_cast<size_t>(head) * dh + d0;   // even
    const uint32_t* dy32 = reinterpret_cast<const uint32_t*>(dY + cb);
    const uint32_t* g32 = reinterpret_cast<const uint32_t*>(gate + cb);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (d0 + 2 * k < dh) {   // dh is even: pairs stay inside the head
        dyw[k] = __ldg(dy32 + k);
        gw[k] = __ldg(g32 + k);
      }
    const size_t ob = (((static_cast<size_t>(b) * H + yp) * W + xp) * heads + head) * DP + d0;
    const uint4 ov = __ldg(reinterpret_cast<const uint4*>(O + ob));
    const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      o[2 * k] = bf16_lo(ow[k]);
      o[2 * k + 1] = bf16_hi(ow[k]);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (d0 + e < dh) {
        const uint32_t pair_dy = dyw[e >> 1], pair_g = gw[e >> 1];
        const float dy = (e & 1) ? bf16_hi(pair_dy) : bf16_lo(pair_dy);
        const float gg = (e & 1) ? bf16_hi(pair_g) : bf16_lo(pair_g);
        v[e] = __bfloat162float(__float2bfloat16_rn(sc * dy * gg));
        dsum = fmaf(v[e], o[e], dsum);
      }
    }
  }
  dsum += __shfl_xor_sync(0xffffffffu, dsum, 1);
  dsum += __shfl_xor_sync(0xffffffffu, dsum, 2);
  if (!in_range) return;
  const __nv_bfloat16 hi = __float2bfloat16_rn(-dsum);
  const __nv_bfloat16 lo = __float2bfloat16_rn(-dsum - __bfloat162float(hi));
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float pair[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int d = d0 + 2 * k + u;
      float x = 0.f;
      if (real) x = d < dh ? v[2 * k + u] : (d == dh ? __bfloat162float(hi) : (d == dh + 1 ? __bfloat162float(lo) : 0.f));
      pair[u] = x;
    }
    w[k] = pack_bf16x2(pair[0], pair[1]);   // exact: every value is already bf16
  }
  reinterpret_cast<uint4*>(dO + th * 32)[g] = make_uint4(w[0], w[1], w[2], w[3]);
  if (dG && real && d0 < dh) {
    uint32_t* dg32 = reinterpret_cast<uint32_t*>(dG + cb);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (d0 + 2 * k < dh) {
        float r[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int e = 2 * k + u;
          const float dy = u ? bf16_hi(dyw[k]) : bf16_lo(dyw[k]);
          const float gg = u ? bf16_hi(gw[k]) : bf16_lo(gw[k]);
          r[u] = dy * o[e] * gg * (1.f - gg);
        }
        dg32[k] = pack_bf16x2(r[0], r[1]);
      }
    }
  }
  if (g == 0) Dsum[((static_cast<size_t>(b) * heads + head) * Hp + yp) * Wp + xp] = dsum / sc;
}

// Q'' of the folded backward, per padded token and head (l2 = s * log2 e):
// content columns bf16(l2 * Qc) with -log2(e) * lse as a bf16 (hi, lo) pair
// in columns dh and dh+1 (zeros past them), rank columns bf16(l2 * Qp) of the
// token's window position.
__global__ void qfold_kernel(const __nv_bfloat16* __restrict__ Qc, const __nv_bfloat16* __restrict__ qp,
                             const float* __restrict__ lse, __nv_bfloat16* __restrict__ Qf, __nv_bfloat16* __restrict__ Qpf,
                             int B, int Hp, int Wp, int heads, int dh, int DP, int M, float sl2) {
  // four threads per (padded token, head), eight columns each
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long total = static_cast<long long>(B) * Hp * Wp * heads;
  const long long th = gid >> 2;
  const int g = static_cast<int>(gid & 3);
  if (th >= total) return;
  const int head = static_cast<int>(th % heads);
  const long long pix = th / heads;
  const int x = static_cast<int>(pix % Wp);
  const int y = static_cast<int>((pix / Wp) % Hp);
  const int b = static_cast<int>(pix / (static_cast<long long>(Wp) * Hp));
  const int d0 = 8 * g;
  if (d0 < DP) {
    // P = exp(s S - lse) = 2^(l2 S - log2(e) lse)
    const float lse2 = lse[((static_cast<size_t>(b) * heads + head) * Hp + y) * Wp + x] * kLog2e;
    const __nv_bfloat16 hi = __float2bfloat16_rn(-lse2);
    const __nv_bfloat16 lo = __float2bfloat16_rn(-lse2 - __bfloat162float(hi));
    const uint4 qv = __ldg(reinterpret_cast<const uint4*>(Qc + th * DP) + g);
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float pair[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int d = d0 + 2 * k + u;
        const float q = u ? bf16_hi(qw[k]) : bf16_lo(qw[k]);
        pair[u] = d < dh ? sl2 * q : (d == dh ? __bfloat162float(hi) : (d == dh + 1 ? __bfloat162float(lo) : 0.f));
      }
      w[k] = pack_bf16x2(pair[0], pair[1]);
    }
    reinterpret_cast<uint4*>(Qf + th * DP)[g] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (d0 < kR) {
    const uint4 cv = __ldg(reinterpret_cast<const uint4*>(qp + ((static_cast<size_t>(head) * M + y % M) * M + x % M) * kR) + g);
    const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = pack_bf16x2(sl2 * bf16_lo(cw[k]), sl2 * bf16_hi(cw[k]));
    reinterpret_cast<uint4*>(Qpf + th * kR)[g] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Sum of per-window partials over the B*nW windows (fixed order: deterministic).
__global__ void window_sum_kernel(const float* __restrict__ part, float* __restrict__ out, int nwin, long long per_win) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= per_win) return;
  float s = 0.f;
  for (int w = 0; w < nwin; ++w) s += part[static_cast<size_t>(w) * per_win + i];
  out[i] = s;
}

bool tiles64(int M, int* tc, int* tr) {
  for (int c = 64; c >= 8; c /= 2) {
    const int r = 64 / c;
    if (M % c == 0 && M % r == 0) {
      *tc = c;
      *tr = r;
      return true;
    }
  }
  return false;
}

// exponential pairs per eight taken by the FMA polynomial instead of MUFU
// (measured at the 96x96 training shape: 1 of 8 in both kernels beats 0, 2,
// 3 and 4 and the mixes 1/2 and 2/1)
#ifndef RIB_BWD_POLY
#define RIB_BWD_POLY 1
#endif

template <int DP, bool FOLD>
cudaError_t launch_bwd_impl(const AttnBwdLaunch& a, cudaStream_t stream) {
  using Lay = BwdLay<DP>;
  const int nwx = (a.W + a.M - 1) / a.M, nwy = (a.H + a.M - 1) / a.M;
  const int Hp = nwy * a.M, Wp = nwx * a.M;
  const int nwin = a.B * nwx * nwy;
  int tc2, tr2;
  if (!tiles64(a.M, &tc2, &tr2)) return cudaErrorInvalidValue;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle swc = DP == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  const uint64_t dimsC[5] = {uint64_t(DP), uint64_t(a.heads), uint64_t(Wp), uint64_t(Hp), uint64_t(a.B)};
  const uint64_t strC[4] = {uint64_t(DP) * 2, uint64_t(a.heads) * DP * 2, uint64_t(Wp) * a.heads * DP * 2,
                            uint64_t(Hp) * Wp * a.heads * DP * 2};
  const uint64_t dimsV[5] = {32u, uint64_t(a.heads), uint64_t(Wp), uint64_t(Hp), uint64_t(a.B)};
  const uint64_t strV[4] = {64u, uint64_t(a.heads) * 64, uint64_t(Wp) * a.heads * 64, uint64_t(Hp) * Wp * a.heads * 64};
  // per-token rank features (the fold's Q''p): [B][Hp][Wp][heads][16]
  const uint64_t dimsT[5] = {uint64_t(kR), uint64_t(a.heads), uint64_t(Wp), uint64_t(Hp), uint64_t(a.B)};
  const uint64_t strT[4] = {uint64_t(kR) * 2, uint64_t(a.heads) * kR * 2, uint64_t(Wp) * a.heads * kR * 2,
                            uint64_t(Hp) * Wp * a.heads * kR * 2};
  const uint64_t dimsP[4] = {uint64_t(kR), uint64_t(a.M), uint64_t(a.M), uint64_t(a.heads)};
  const uint64_t strP[3] = {uint64_t(kR) * 2, uint64_t(a.M) * kR * 2, uint64_t(a.M) * a.M * kR * 2};
  const uint64_t dimsL[4] = {uint64_t(Wp), uint64_t(Hp), uint64_t(a.heads), uint64_t(a.B)};
  const uint64_t strL[3] = {uint64_t(Wp) * 4, uint64_t(Hp) * Wp * 4, uint64_t(a.heads) * Hp * Wp * 4};
  auto box5 = [&](int w0, int tc, int tr, uint32_t (&bx)[5]) { bx[0] = w0; bx[1] = 1; bx[2] = tc; bx[3] = tr; bx[4] = 1; };
  uint32_t b128C[5], b64C[5], b128V[5], b64V[5], b128T[5], b64T[5];
  box5(DP, a.tc, a.tr, b128C);
  box5(DP, tc2, tr2, b64C);
  box5(32, a.tc, a.tr, b128V);
  box5(32, tc2, tr2, b64V);
  box5(kR, a.tc, a.tr, b128T);
  box5(kR, tc2, tr2, b64T);
  const uint32_t b128P[4] = {uint32_t(kR), uint32_t(a.tc), uint32_t(a.tr), 1u};
  const uint32_t b64P[4] = {uint32_t(kR), uint32_t(tc2), uint32_t(tr2), 1u};
  const uint32_t b64L[4] = {uint32_t(tc2), uint32_t(tr2), 1u, 1u};
  // the streamed side (dQ: Kc, Kp; dK/dV: Q'') in 8-feature atoms (16-byte rows, no swizzle)
  uint32_t b64A[5];
  box5(8, tc2, tr2, b64A);
  const uint32_t b64PA[4] = {8u, uint32_t(tc2), uint32_t(tr2), 1u};

  BwdParams p;
  p.B = a.B; p.heads = a.heads; p.dh = a.dh; p.M = a.M; p.Hp = Hp; p.Wp = Wp; p.nwx = nwx; p.nwy = nwy;
  p.tc = a.tc; p.tr = a.tr; p.tiles_x = a.M / a.tc;
  p.tc2 = tc2; p.tr2 = tr2; p.tiles_x2 = a.M / tc2;
  p.n_stream = (a.M * a.M) / 64;
  p.n_own = (a.M * a.M) / 128;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.scale = a.scale;
  p.inv_scale = 1.f / a.scale;
  p.inv_scale_log2 = 1.f / p.scale_log2;
  p.lse = a.lse;
  p.err = device_error_word();
  const long long units = static_cast<long long>(nwin) * a.heads * p.n_own;
  if (units <= 0) return cudaSuccess;

  // the Q side of the S products: Q'' (fold, written here) or the stored Qc and the cache
  const void* qc_src = a.Qc;
  const void* qp_src = a.qp;
  if (FOLD) {
    const long long total = static_cast<long long>(a.B) * Hp * Wp * a.heads;
    qfold_kernel<<<static_cast<unsigned>((4 * total + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a.Qc), static_cast<const __nv_bfloat16*>(a.qp), a.lse,
        static_cast<__nv_bfloat16*>(a.qf), static_cast<__nv_bfloat16*>(a.qpf), a.B, Hp, Wp, a.heads, a.dh, DP, a.M,
        p.scale_log2);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    qc_src = a.qf;
    qp_src = a.qpf;
  }
  auto encode_qp = [&](CUtensorMap* m, bool own) {
    if (FOLD) return encode_tiled(m, bf, 5, const_cast<void*>(qp_src), dimsT, strT, own ? b128T : b64T, CU_TENSOR_MAP_SWIZZLE_32B);
    return encode_tiled(m, bf, 4, const_cast<void*>(qp_src), dimsP, strP, own ? b128P : b64P, CU_TENSOR_MAP_SWIZZLE_32B);
  };

  // dQ: own = Q tile (Q, Qp, dO''), streamed = K tiles (Kc, Kp, V)
  {
    CUtensorMap tq, tqp, tdo, tk, tkp, tv;
    if (encode_tiled(&tq, bf, 5, const_cast<void*>(qc_src), dimsC, strC, b128C, swc) != CUDA_SUCCESS ||
        encode_qp(&tqp, true) != CUDA_SUCCESS ||
        encode_tiled(&tdo, bf, 5, const_cast<void*>(a.dO), dimsV, strV, b128V, CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS ||
        encode_tiled(&tk, bf, 5, const_cast<void*>(a.Kc), dimsC, strC, b64A, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS ||
        encode_tiled(&tkp, bf, 4, const_cast<void*>(a.kp), dimsP, strP, b64PA, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS ||
        encode_tiled(&tv, bf, 5, const_cast<void*>(a.V), dimsV, strV, b64V, CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    BwdParams pq = p;
    pq.out_c = a.dQc;
    pq.out_v = nullptr;
    pq.out_p = a.ws_q;
    auto kern = rib_attn_bwd_dq_kernel<DP, FOLD, RIB_BWD_POLY>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::ALLOC);
    if (e != cudaSuccess) return e;
    kern<<<static_cast<unsigned>(units), kBwdThreads, Lay::ALLOC, stream>>>(tq, tqp, tdo, tk, tkp, tv, pq);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // dK/dV: own = K tile (Kc, Kp, V), streamed = Q tiles (Q, Qp, dO'', and lse without the fold)
  {
    CUtensorMap tk, tkp, tv, tq, tqp, tdo, tl;
    if (encode_tiled(&tk, bf, 5, const_cast<void*>(a.Kc), dimsC, strC, b128C, swc) != CUDA_SUCCESS ||
        encode_tiled(&tkp, bf, 4, const_cast<void*>(a.kp), dimsP, strP, b128P, CU_TENSOR_MAP_SWIZZLE_32B) != CUDA_SUCCESS ||
        encode_tiled(&tv, bf, 5, const_cast<void*>(a.V), dimsV, strV, b128V, CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS ||
        encode_tiled(&tq, bf, 5, const_cast<void*>(qc_src), dimsC, strC, b64A, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS ||
        (FOLD ? encode_tiled(&tqp, bf, 5, const_cast<void*>(qp_src), dimsT, strT, b64A, CU_TENSOR_MAP_SWIZZLE_NONE)
              : encode_tiled(&tqp, bf, 4, const_cast<void*>(qp_src), dimsP, strP, b64PA, CU_TENSOR_MAP_SWIZZLE_NONE)) !=
            CUDA_SUCCESS ||
        encode_tiled(&tdo, bf, 5, const_cast<void*>(a.dO), dimsV, strV, b64V, CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS ||
        encode_tiled(&tl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(a.lse), dimsL, strL, b64L,
                     CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    BwdParams pk = p;
    pk.out_c = a.dKc;
    pk.out_v = a.dV;
    pk.out_p = a.ws_k;
    auto kern = rib_attn_bwd_dkv_kernel<DP, FOLD, RIB_BWD_POLY>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::ALLOC);
    if (e != cudaSuccess) return e;
    kern<<<static_cast<unsigned>(units), kBwdThreads, Lay::ALLOC, stream>>>(tk, tkp, tv, tq, tqp, tdo, tl, pk);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // dQp, dKp: sums over the windows
  const long long per_win = static_cast<long long>(a.heads) * a.M * a.M * kR;
  const unsigned blocks = static_cast<unsigned>((per_win + 255) / 256);
  window_sum_kernel<<<blocks, 256, 0, stream>>>(a.ws_q, a.dQp, nwin, per_win);
  window_sum_kernel<<<blocks, 256, 0, stream>>>(a.ws_k, a.dKp, nwin, per_win);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_window_attention_bwd(const AttnBwdLaunch& a, cudaStream_t stream) {
  // the lse rides in the score product when the padded head has two spare columns
  const bool fold = a.dh + 2 <= a.DP;
  if (a.DP == 32) return fold ? launch_bwd_impl<32, true>(a, stream) : launch_bwd_impl<32, false>(a, stream);
  return fold ? launch_bwd_impl<16, true>(a, stream) : launch_bwd_impl<16, false>(a, stream);
}

cudaError_t launch_bwd_prep(const void* dY, const void* gate, const void* O, void* dO, float* Dsum, void* dG, int B,
                            int H, int W, int C, int heads, int M, float scale, cudaStream_t stream) {
  const int Hp = (H + M - 1) / M * M, Wp = (W + M - 1) / M * M;
  const long long total = static_cast<long long>(B) * Hp * Wp * heads;
  if (total == 0) return cudaSuccess;
  bwd_prep_kernel<<<static_cast<unsigned>((4 * total + 255) / 256), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(dY), static_cast<const __nv_bfloat16*>(gate),
      static_cast<const __nv_bfloat16*>(O), static_cast<__nv_bfloat16*>(dO), Dsum, static_cast<__nv_bfloat16*>(dG), B, H, W,
      C, heads, Hp, Wp, scale);
  return cudaGetLastError();
}

}  // namespace rib
