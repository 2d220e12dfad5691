// Fused windowed RIB attention forward for sm_100a.
//
// What it computes (RIB/SST write-up, section 2.2 "注意力计算重构" and section
// 2.3 CLA): for every non-overlapping M x M window and head,
//   S = Qc Kc^T + Qp Kp^T          (Qc carries 1/sqrt(dh), Qp carries 1/sqrt(R))
//   O = softmax(softmax_scale * S) V,   Y = O * sigmoid(G) (+ residual)
// The concatenation [Qc, Qp][Kc, Kp]^T is realised as two tensor-core
// products accumulating into the same TMEM tile (content part K = DP, then the
// rank part K = R), so no N x N matrix ever reaches memory.
//
// Inputs are in the window-padded layout [B][Hp][Wp][heads][*] written by the
// projection: Qc, Kc bf16 (DP columns), V bf16 (DPV = 32 columns) whose
// column dh is 1 for every token, padded ones included. P is produced as
// bf16 by the exponentials and P.V accumulates in fp32 TMEM, so column dh of
// the accumulator is the softmax denominator, summed by the tensor core from
// the very P values that weight V.
//
// One CTA owns one 128-query tile of one (window, head) and streams the
// window's keys in BK-token tiles (BK = 64 on the launch path; the kernel
// also takes 128); four CTAs share an SM, so each SM sub-partition runs the
// softmax warps of several independent tiles and one tile's MMA and barrier
// latencies hide behind the exponentials of the others.
//   warp 0      TMA producer: the Q tile once, then Kc / Kp / V tiles into a
//               ring of NS shared-memory stages (window partition by TMA box
//               coordinates), each stage refilled once both products of its
//               tile are done; also the issuer of the P(j).V(j) products once
//               P(j) is in TMEM (a thread's tcgen05.mma instructions run one
//               after another, so QK and P.V go out from separate threads).
//   warp 1      TMEM owner and QK issuer: QK(j+1) as soon as the softmax has
//               read S(j).
//   warps 2-5   softmax, thread = query row: reads its S row from TMEM,
//               exponentiates in registers (exp2 domain) and writes P (bf16)
//               back to TMEM for the P.V product (A operand from TMEM).
// The epilogue multiplies by the gate and stores straight to the image layout
// [B][H][W][C] (window reverse + crop in the store).
//
// Softmax in the score product (heads with dh < DP, the default path). The
// content tiles have spare columns d >= dh; the projection writes Kc[dh] = 1
// for every key. The first key tile's scores give each row a reference m (the
// bf16-rounded maximum of that tile's scaled scores); each softmax thread then
// rewrites its row of the Q tile in shared memory as
//     Q'[d] = bf16(scale_log2 * Q[d])  (content and rank columns),  Q'[dh] = -m
// and the first tile's QK is issued again, so for every key tile the tensor
// core delivers x = scale_log2 * S - m directly and the per-score work is one
// exponential (MUFU ex2, or the FMA-pipe cubic for POLY of every 8 pairs) and
// half a bf16 pack: no running maximum, no scale and subtract. The row is read
// from TMEM in 16-column chunks, the next chunk loading while the current one
// is exponentiated (S is released once its last chunk is in registers), which
// keeps the live registers within the four-CTAs-per-SM budget. m stays fixed for the row (O
// and its ones-column denominator accumulate with the same reference, which
// cancels in O / l), and bf16 P leaves 2^127 of headroom above the first
// tile's maximum. A row
// whose denominator reaches 2^100 (or overflows) is the only case where that
// headroom can have been exceeded; if any row of the tile gets there, the CTA
// discards the pass and runs the tile again with the safe softmax below.
//
// Safe softmax (dh == DP, the key-padding mask, and the re-run): the row
// maximum of every tile, a running reference that is kept until a tile's
// maximum exceeds it by more than 2^8 (then O is rescaled in TMEM before the
// next P is released), and x = scale_log2 * S - m by one packed FMA per pair.
//
// TMEM columns: S at 0 (BK fp32), P at BK (BK/2 columns of bf16 pairs), the
// O accumulator at 3BK/2 (32).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rib_internal.h"
#include "sm100.cuh"

namespace rib {

namespace {

// exponential pairs (of every 8) computed on the FMA pipe, per block shape
// (measured at 640x360, window 64: 2 of 8 is fastest for the 64-key shape)
#ifndef RIB_ATTN_POLY_SMALL
#define RIB_ATTN_POLY_SMALL 2
#endif
// columns of S read from TMEM at a time by the folded softmax (16, 32 or 64)
#ifndef RIB_ATTN_FOLD_CHUNK
#define RIB_ATTN_FOLD_CHUNK 16
#endif
// CTAs per SM of the 64-key-tile shape
#ifndef RIB_ATTN_MINB_SMALL
#define RIB_ATTN_MINB_SMALL 4
#endif

constexpr int kBQ = 128;       // queries per tile
constexpr int kR = 16;         // rank of the positional features
constexpr int kThreads = 192;  // producer, issuer, four softmax warps
constexpr float kLn2 = 0.6931471805599453f;
// a denominator at or above 2^100 (or not finite) makes the tile re-run
// with the safe softmax
constexpr float kRedoDenominator = 1.2676506002282294e30f;

// TMEM columns of one CTA: S (BK), P (BK/2) and O (32), rounded up to the
// power of two the allocator takes.
__host__ __device__ constexpr int attn_tmem_cols(int BK) { return BK + BK / 2 + 32 <= 128 ? 128 : 256; }

struct AttnParams {
  int B, H, W, C, heads, dh, M, tc, tr, tiles_x, n_tiles, nwx, nwy, Hp, Wp;
  int tck, trk, tiles_xk, n_kv;   // key tiles: tck x trk tokens, n_kv per window
  float scale_log2;
  const __nv_bfloat16* gate;
  const void* resid;   // bf16, fp32 (out_f32) or fp16 (out_f16) [B][H][W][C]
  void* Y;             // bf16, fp32 (out_f32) or fp16 (out_f16) [B][H][W][C]
  int out_f32, out_f16;
  float* lse;
  __nv_bfloat16* O_out;
  int* err;
};

template <int DP, int NS, int BK, int DPV = 32>
struct Layout {
  static constexpr int QC = kBQ * DP * 2;   // bytes of the content tile
  static constexpr int QP = kBQ * kR * 2;   // bytes of the rank tile
  static constexpr int KC = BK * DP * 2;
  static constexpr int KP = BK * kR * 2;
  static constexpr int VB = BK * DPV * 2;
  static constexpr int STAGE = KC + KP + VB;
  static constexpr int OFF_QC = 0;
  static constexpr int OFF_QP = OFF_QC + QC;
  static constexpr int OFF_ST = OFF_QP + QP;
  static constexpr int OFF_BAR = OFF_ST + NS * STAGE;
  // barriers: q_full, kv_full[NS], kv_empty[NS], s_full, s_free, p_full, pv_full, done
  static constexpr int NBAR = 1 + 2 * NS + 5;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // misc words: TMEM base, abort flag, teardown abort word, re-run flag
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;   // slack for 1024-byte alignment
  // content tiles: rows of DP bf16 = 64 B (SW64) or 32 B (SW32)
  static constexpr uint32_t SW_C = DP == 32 ? SW_64B : SW_32B;
  static constexpr uint32_t SBO_C = 8 * DP * 2;
  // V tiles: rows of DPV bf16 = 64 B (SW64)
  static constexpr uint32_t SW_V = SW_64B;
  static constexpr uint32_t SBO_V = 8 * DPV * 2;
};

enum WaitSite : int {
  SITE_Q = 101, SITE_KV_EMPTY = 102, SITE_KV_FULL = 103, SITE_S_FREE = 104, SITE_P_FULL = 105,
  SITE_S_FULL = 106, SITE_PV_FULL = 107, SITE_DONE = 108, SITE_DRAIN = 109,
};

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// OR of a predicate over the n threads of named barrier `id` (all of which
// must reach it).
__device__ __forceinline__ bool named_any(int id, int n, bool v) {
  uint32_t r;
  asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
               : "=r"(r) : "r"(v ? 1u : 0u), "r"(id), "r"(n) : "memory");
  return r != 0;
}

// Rewrites row r of the shared-memory Q tile (content then rank part, as the
// TMA wrote them: 64-byte rows with the 64B swizzle for DP = 32, 32-byte rows
// with the 32B swizzle for DP = 16 and the rank part) as bf16(sl2 * Q), with
// content column dh set to neg_m.
template <int DP>
__device__ __forceinline__ void fold_q_row(uint8_t* qc, uint8_t* qp, int r, int dh, float sl2, float neg_m) {
  auto scale_chunk = [&](uint4* ptr, int d0) {
    const uint4 v = *ptr;
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = (d0 + 2 * e == dh) ? neg_m : bf16_lo(w[e]) * sl2;
      w[e] = pack_bf16x2(lo, bf16_hi(w[e]) * sl2);
    }
    *ptr = make_uint4(w[0], w[1], w[2], w[3]);
  };
#pragma unroll
  for (int c = 0; c < DP / 8; ++c) {
    const int pc = DP == 32 ? (c ^ ((r >> 1) & 3)) : (c ^ ((r >> 2) & 1));
    scale_chunk(reinterpret_cast<uint4*>(qc + r * DP * 2 + pc * 16), 8 * c);
  }
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int pc = c ^ ((r >> 2) & 1);
    scale_chunk(reinterpret_cast<uint4*>(qp + r * kR * 2 + pc * 16), -1000);   // no column is dh here
  }
}

// POLY of every 8 exponential pairs run on the FMA pipe, the rest on MUFU;
// MINB CTAs per SM; MASK compiles in the key-padding mask (a separate
// instantiation, so the default path carries none of its code); FOLD runs the
// softmax in the score product (first pass) with the safe softmax as the
// re-run.
template <int DP, int NS, int POLY, int BK, int MINB, bool MASK, bool FOLD>
__global__ void __launch_bounds__(kThreads, MINB)
rib_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_qp,
                    const __grid_constant__ CUtensorMap tm_kp, const AttnParams p) {
  static_assert(!(MASK && FOLD), "the key-padding mask runs the safe softmax");
  using Lay = Layout<DP, NS, BK>;
  constexpr uint32_t kCols = attn_tmem_cols(BK);
  constexpr uint32_t kColP = BK;
  constexpr uint32_t kColO = BK + BK / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = bars + 1 + NS;
  uint64_t* s_full = bars + 1 + 2 * NS;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_full = s_full + 3;
  uint64_t* done = s_full + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + Lay::OFF_MISC + 4);
  volatile uint32_t* redo_flag = reinterpret_cast<volatile uint32_t*>(smem + Lay::OFF_MISC + 12);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // work unit -> (b, wy, wx, head, query tile)
  int u = blockIdx.x;
  const int qt = u % p.n_tiles;
  u /= p.n_tiles;
  const int head = u % p.heads;
  const int w = u / p.heads;
  const int wx = w % p.nwx;
  const int wy = (w / p.nwx) % p.nwy;
  const int b = w / (p.nwx * p.nwy);
  const int y0 = wy * p.M, x0 = wx * p.M;
  const int n_kv = p.n_kv;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 2);   // the QK (warp 1) and P.V (warp 0) products of the tile
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(p_full, 4);
    mbar_init(pv_full, 1);
    mbar_init(done, 2);
    *abort_flag = 0u;
    tmem_holder[2] = 0u;   // abort word of the teardown drains (never raised by others)
    *redo_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, p.err};

  // Pass 0: the folded softmax (FOLD) or the safe one; pass 1 (FOLD only, when
  // a row of pass 0 reached the re-run threshold): the safe softmax. Barrier
  // phases continue across the passes (tile jg = pass * n_kv + j).
  for (int pass = 0; pass < (FOLD ? 2 : 1); ++pass) {
    const int j0 = pass * n_kv;
    const bool fold = FOLD && pass == 0;
    // phases of s_full / s_free before this pass: the folded pass completes
    // them n_kv + 1 times (tile 0 twice), the safe pass n_kv times
    const int sph = pass == 0 ? 0 : n_kv + 1;
    const uint32_t sst = smem_u32(smem + Lay::OFF_ST);
    const uint32_t tS = tmem;
    const uint32_t tP = tmem + kColP;
    const uint32_t tO = tmem + kColO;
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      // and P.V issuer: a thread's tcgen05.mma instructions run one after
      // another, so the P.V products go out from this thread while warp 1
      // issues the QK products; each tile's stage is refilled once both of
      // its products are done
      if (lane == 0) {
        if (pass == 0) {
          tma_prefetch_desc(&tm_q);
          tma_prefetch_desc(&tm_k);
          tma_prefetch_desc(&tm_v);
          tma_prefetch_desc(&tm_qp);
          tma_prefetch_desc(&tm_kp);
        }
        mbar_arrive_expect_tx(q_full, Lay::QC + Lay::QP);
        {
          const int ty = (qt / p.tiles_x) * p.tr, tx = (qt % p.tiles_x) * p.tc;
          tma_load_5d(smem + Lay::OFF_QC, &tm_q, q_full, 0, head, x0 + tx, y0 + ty, b);
          tma_load_4d(smem + Lay::OFF_QP, &tm_qp, q_full, 0, tx, ty, head);
        }
        int issued = 0;
        bool ok = true;
        // key tile i into its stage, once the stage's previous tile is done
        auto load_kv = [&](int i) {
          const int ig = j0 + i, st = ig % NS;
          if (ig >= NS && !mbar_wait(&kv_empty[st], ((ig / NS) - 1) & 1, wc, SITE_KV_EMPTY)) return false;
          uint8_t* sb = smem + Lay::OFF_ST + st * Lay::STAGE;
          const int ty = (i / p.tiles_xk) * p.trk, tx = (i % p.tiles_xk) * p.tck;
          mbar_arrive_expect_tx(&kv_full[st], Lay::STAGE);
          tma_load_5d(sb, &tm_k, &kv_full[st], 0, head, x0 + tx, y0 + ty, b);
          tma_load_4d(sb + Lay::KC, &tm_kp, &kv_full[st], 0, tx, ty, head);
          tma_load_5d(sb + Lay::KC + Lay::KP, &tm_v, &kv_full[st], 0, head, x0 + tx, y0 + ty, b);
          issued = i + 1;
          return true;
        };
        constexpr uint32_t idesc_pv = idesc_bf16(128, 32, false, true);
        for (int i = 0; ok && i < NS && i < n_kv; ++i) ok = load_kv(i);
        for (int j = 0; ok && j < n_kv; ++j) {
          const int jg = j0 + j;
          if (!(ok = mbar_wait(p_full, jg & 1, wc, SITE_P_FULL))) break;
          tc_fence_after();
          const uint32_t vb = sst + (jg % NS) * Lay::STAGE + Lay::KC + Lay::KP;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // MN-major V: 16 keys per MMA = 16 rows of DPV bf16
            umma_ts(tO, tP + 8u * k, make_sdesc(vb + k * 16 * 32 * 2, Lay::VB, Lay::SBO_V, Lay::SW_V), idesc_pv,
                    (j > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(pv_full);
          umma_commit(&kv_empty[jg % NS]);
          if (j + NS < n_kv) ok = load_kv(j + NS);
        }
        umma_commit(done);
        // Drain: every copy issued in this pass has landed and every P.V
        // product has completed before the CTA may exit or start the next pass.
        const WaitCtx drain{reinterpret_cast<volatile uint32_t*>(tmem_holder + 2), p.err};
        mbar_wait(q_full, pass & 1, drain, SITE_DRAIN);
        for (int i = issued - NS > 0 ? issued - NS : 0; i < issued; ++i)
          mbar_wait(&kv_full[(j0 + i) % NS], ((j0 + i) / NS) & 1, drain, SITE_DRAIN);
        mbar_wait(done, pass & 1, drain, SITE_DONE);
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- QK issuer
      if (lane == 0) {
        constexpr uint32_t idesc_qk = idesc_bf16(128, BK, false, false);
        const uint32_t sq = smem_u32(smem + Lay::OFF_QC);
        const uint32_t sqp = smem_u32(smem + Lay::OFF_QP);
        auto issue_qk = [&](int st) {
          const uint32_t b0 = sst + st * Lay::STAGE;
#pragma unroll
          for (int k = 0; k < DP / 16; ++k) {
            umma_ss(tS, make_sdesc(sq + 32 * k, 16, Lay::SBO_C, Lay::SW_C),
                    make_sdesc(b0 + 32 * k, 16, Lay::SBO_C, Lay::SW_C), idesc_qk, k > 0 ? 1u : 0u);
          }
          umma_ss(tS, make_sdesc(sqp, 16, 256, SW_32B), make_sdesc(b0 + Lay::KC, 16, 256, SW_32B), idesc_qk, 1u);
          umma_commit(s_full);
        };
        bool ok = mbar_wait(q_full, pass & 1, wc, SITE_Q) && mbar_wait(&kv_full[j0 % NS], (j0 / NS) & 1, wc, SITE_KV_FULL);
        if (ok) {
          tc_fence_after();
          issue_qk(j0 % NS);
        }
        if (ok && fold) {
          // tile 0 again, once the softmax has read its raw scores and
          // rewritten the Q tile with the scale and the row references
          if ((ok = mbar_wait(s_free, sph & 1, wc, SITE_S_FREE))) {
            tc_fence_after();
            issue_qk(j0 % NS);
          }
        }
        if (ok) umma_commit(&kv_empty[j0 % NS]);
        const int sp0 = sph + (fold ? 1 : 0);   // S phase of tile 0 in this pass
        for (int j = 0; ok && j + 1 < n_kv; ++j) {
          const int jg = j0 + j;
          const int st1 = (jg + 1) % NS;
          if (!(ok = mbar_wait(&kv_full[st1], ((jg + 1) / NS) & 1, wc, SITE_KV_FULL))) break;
          if (!(ok = mbar_wait(s_free, (sp0 + j) & 1, wc, SITE_S_FREE))) break;
          tc_fence_after();
          issue_qk(st1);
          umma_commit(&kv_empty[st1]);
        }
        // every MMA issued above completes before the pass ends
        umma_commit(done);
        const WaitCtx drain{reinterpret_cast<volatile uint32_t*>(tmem_holder + 2), p.err};
        mbar_wait(done, pass & 1, drain, SITE_DONE);
      }
    } else {
      // ---------------------------------------------------------- softmax
      const int quarter = warp & 3;             // TMEM lane quarter this warp may access
      const int row = quarter * 32 + lane;      // query row inside the tile
      const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t tS = tmem + lane_off;
      const uint32_t tP = tmem + lane_off + kColP;
      const uint32_t tO = tmem + lane_off + kColO;
      const float sl2 = p.scale_log2;

      // row maximum: independent 3-input max chains
      auto chain_max = [](const uint32_t (&v)[32]) {
        float a = fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
        for (int i = 3; i + 1 < 32; i += 2) a = fmax3(a, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
        return fmaxf(a, __uint_as_float(v[31]));
      };
      // P = 2^(scale_log2 * S - m) of one 32-column chunk, into TMEM
      auto exp_chunk_scaled = [&](const uint32_t (&sv)[32], uint32_t col, float m_ref) {
        const uint64_t scale2 = f2_pack(sl2, sl2);
        const uint64_t negm2 = f2_pack(-m_ref, -m_ref);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint64_t x = f2_fma(f2_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), scale2, negm2);
          float x0, x1;
          f2_unpack(x, x0, x1);
          pk[i] = ((i & 7) < POLY) ? exp2_poly_bf16x2(x0, x1) : pack_bf16x2(ex2_approx(x0), ex2_approx(x1));
        }
        tmem_st16(tP + col, pk);
      };
      float m = -INFINITY;
      bool ok = true;
      if (fold) {
        constexpr int NC = BK / 32;   // 32-column chunks of the S row
        // tile 0, raw scores: the row's reference, exactly representable in
        // the bf16 Q column that carries it into every later score
        ok = warp_all(mbar_wait(s_full, sph & 1, wc, SITE_S_FULL));
        if (ok) {
          tc_fence_after();
          float mx = -INFINITY;
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            uint32_t sv[32];
            tmem_ld32(tS + 32 * c, sv);
            tmem_wait_ld();
            mx = fmaxf(mx, chain_max(sv));
          }
          m = __bfloat162float(__float2bfloat16_rn(mx * sl2));
          fold_q_row<DP>(smem + Lay::OFF_QC, smem + Lay::OFF_QP, row, p.dh, sl2, -m);
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free);
        }
        // CH-column chunks of the S row, the next one loading while the
        // current one is exponentiated
        constexpr int CH = RIB_ATTN_FOLD_CHUNK < BK ? RIB_ATTN_FOLD_CHUNK : BK;
        constexpr int NCH = BK / CH;
        for (int j = 0; ok && j < n_kv; ++j) {
          const int jg = j0 + j;
          ok = warp_all(mbar_wait(s_full, (sph + 1 + j) & 1, wc, SITE_S_FULL));
          if (!ok) break;
          tc_fence_after();
          uint32_t sa[CH], sb[CH];
          tmem_ld_cols<CH>(tS, sa);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            uint32_t (&cur)[CH] = (c & 1) ? sb : sa;
            uint32_t (&nxt)[CH] = (c & 1) ? sa : sb;
            if (c + 1 < NCH) {
              tmem_ld_cols<CH>(tS + CH * (c + 1), nxt);
            } else {
              // the whole row has been read: the next QK may overwrite S
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(s_free);
            }
#pragma unroll
            for (int h = 0; h < CH / 16; ++h) {
              uint32_t pk[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float x0 = __uint_as_float(cur[16 * h + 2 * i]), x1 = __uint_as_float(cur[16 * h + 2 * i + 1]);
                pk[i] = (i < POLY) ? exp2_poly_bf16x2(x0, x1) : pack_bf16x2(ex2_approx(x0), ex2_approx(x1));
              }
              if (c == 0 && h == 0 && j > 0) {
                // P.V of the previous tile done before P is overwritten (its
                // latency hides behind the first exponentials); on a timeout
                // the stores below still go to this CTA's own TMEM
                ok = warp_all(mbar_wait(pv_full, (jg - 1) & 1, wc, SITE_PV_FULL));
                tc_fence_after();
              }
              tmem_st8(tP + (CH / 2) * c + 8 * h, pk);
            }
            if (c + 1 < NCH) tmem_wait_ld();
          }
          if (!ok) break;
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full);
        }
      } else {
        // key-padding mask: only windows that reach into the padding need it
        const bool edge = MASK && (y0 + p.M > p.H || x0 + p.M > p.W);
        for (int j = 0; j < n_kv; ++j) {
          const int jg = j0 + j;
          ok = warp_all(mbar_wait(s_full, (sph + j) & 1, wc, SITE_S_FULL));
          if (!ok) break;
          tc_fence_after();
          // the S row in 32-column chunks (s2, s3 only for 128-key tiles)
          uint32_t s0[32], s1[32], s2[32], s3[32];
          tmem_ld32(tS, s0);
          tmem_ld32(tS + 32, s1);
          if constexpr (BK == 128) {
            tmem_ld32(tS + 64, s2);
            tmem_ld32(tS + 96, s3);
          }
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free);
          if (MASK && edge) {
            // column k of the key tile is key (k / tck, k % tck) of the tile at
            // (ky, kx) of the window; padded keys get a -inf score (P = 0). Key
            // tile 0 starts at the window origin, which is always a real pixel,
            // so the running maximum is finite from the first tile on.
            const int yk = y0 + (j / p.tiles_xk) * p.trk, xk = x0 + (j % p.tiles_xk) * p.tck;
            auto mask_chunk = [&](uint32_t (&v)[32], int k0) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int k = k0 + i, yr = k / p.tck;
                if (yk + yr >= p.H || xk + (k - yr * p.tck) >= p.W) v[i] = 0xff800000u;
              }
            };
            mask_chunk(s0, 0);
            mask_chunk(s1, 32);
            if constexpr (BK == 128) {
              mask_chunk(s2, 64);
              mask_chunk(s3, 96);
            }
          }
          float mx;
          if constexpr (BK == 128) mx = fmaxf(fmax3(chain_max(s0), chain_max(s1), chain_max(s2)), chain_max(s3));
          else mx = fmaxf(chain_max(s0), chain_max(s1));
          // Lazy running maximum: keep the reference m unless the tile's maximum
          // exceeds it by more than 2^8 (P then stays <= 256); only then rescale
          // the O accumulator (its ones column, the running denominator, with it).
          const float mt = mx * sl2;
          const float m_new = (mt > m + 8.f) ? mt : m;
          const float alpha = ex2_approx(m - m_new);   // 0 on the first tile, 1 when m is kept

          if (j > 0) {
            // P.V of the previous tile done: P may be overwritten, O is stable
            ok = warp_all(mbar_wait(pv_full, (jg - 1) & 1, wc, SITE_PV_FULL));
            if (!ok) break;
            tc_fence_after();
          }
          exp_chunk_scaled(s0, 0, m_new);
          exp_chunk_scaled(s1, 16, m_new);
          if constexpr (BK == 128) {
            exp_chunk_scaled(s2, 32, m_new);
            exp_chunk_scaled(s3, 48, m_new);
          }
          if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {   // two 16-column halves keep the register peak low
              uint32_t ov[16];
              tmem_ld16(tO + 16u * h, ov);
              tmem_wait_ld();
#pragma unroll
              for (int d = 0; d < 16; ++d) ov[d] = __float_as_uint(__uint_as_float(ov[d]) * alpha);
              tmem_st16(tO + 16u * h, ov);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full);
          m = m_new;
        }
      }
      float o[32];
      if (ok) {
        ok = warp_all(mbar_wait(pv_full, (j0 + n_kv - 1) & 1, wc, SITE_PV_FULL));
        if (ok) {
          tc_fence_after();
          uint32_t ov[32];
          tmem_ld32(tO, ov);
          tmem_wait_ld();
#pragma unroll
          for (int d = 0; d < 32; ++d) o[d] = __uint_as_float(ov[d]);
        }
      }
      float l = 0.f;   // the ones column of V accumulated the denominator
      if (ok) {
#pragma unroll
        for (int d = 0; d < 32; ++d) l = (d == p.dh) ? o[d] : l;
      }
      bool redo = false;
      if (fold) {
        // any row of the tile at the threshold (or not finite): re-run the tile
        float z = 0.f;
#pragma unroll
        for (int d = 0; d < 32; ++d) z += o[d] * 0.f;   // NaN if any O is not finite
        const bool bad = ok && (!(l < kRedoDenominator) || z != 0.f);
        redo = named_any(1, 128, bad);
        if (redo && row == 0) *redo_flag = 1u;
      }
      if (ok && !redo) {
        // ---------------------------------------------------- epilogue
        const float inv_l = 1.f / l;
        const int yy = (qt / p.tiles_x) * p.tr + row / p.tc;
        const int xx = (qt % p.tiles_x) * p.tc + row % p.tc;
        const int y = y0 + yy, x = x0 + xx;
        if (p.lse) p.lse[((static_cast<size_t>(b) * p.heads + head) * p.Hp + y) * p.Wp + x] = (m + __log2f(l)) * kLn2;
        if (y < p.H && x < p.W) {
          const size_t pix = (static_cast<size_t>(b) * p.H + y) * p.W + x;
          const size_t cbase = pix * p.C + static_cast<size_t>(head) * p.dh;
          const uint32_t* g = p.gate ? reinterpret_cast<const uint32_t*>(p.gate + cbase) : nullptr;
          if (p.out_f32) {
            // fp32 residual stream: Y (and the residual) in fp32
            const float2* rs = p.resid ? reinterpret_cast<const float2*>(static_cast<const float*>(p.resid) + cbase)
                                       : nullptr;
            float2* yo = reinterpret_cast<float2*>(static_cast<float*>(p.Y) + cbase);
#pragma unroll
            for (int d = 0; d < DP; d += 2) {
              if (d < p.dh) {
                float v0 = o[d] * inv_l, v1 = o[d + 1] * inv_l;
                if (g) {
                  const uint32_t gv = __ldg(g + d / 2);
                  v0 *= bf16_lo(gv);
                  v1 *= bf16_hi(gv);
                }
                if (rs) {
                  const float2 rv = rs[d / 2];
                  v0 += rv.x;
                  v1 += rv.y;
                }
                yo[d / 2] = make_float2(v0, v1);
              }
            }
          } else {
            // 16-bit Y (and residual): bf16, or fp16 (saturating) for the fp16 path
            const uint32_t* rs = p.resid ? reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(p.resid) + cbase)
                                         : nullptr;
            uint32_t* yo = reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.Y) + cbase);
#pragma unroll
            for (int d = 0; d < DP; d += 2) {
              if (d < p.dh) {
                float v0 = o[d] * inv_l, v1 = o[d + 1] * inv_l;
                if (g) {
                  const uint32_t gv = __ldg(g + d / 2);
                  v0 *= bf16_lo(gv);
                  v1 *= bf16_hi(gv);
                }
                if (rs) {
                  const uint32_t rv = rs[d / 2];
                  v0 += p.out_f16 ? f16_lo(rv) : bf16_lo(rv);
                  v1 += p.out_f16 ? f16_hi(rv) : bf16_hi(rv);
                }
                yo[d / 2] = p.out_f16 ? pack_f16x2_sat(v0, v1) : pack_bf16x2(v0, v1);
              }
            }
          }
          if (p.O_out) {
            uint4* oo = reinterpret_cast<uint4*>(p.O_out + (pix * p.heads + head) * DP);
#pragma unroll
            for (int d = 0; d < DP; d += 8) {
              float w8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) w8[e] = (d + e < p.dh) ? o[d + e] * inv_l : 0.f;
              oo[d / 8] = make_uint4(pack_bf16x2(w8[0], w8[1]), pack_bf16x2(w8[2], w8[3]), pack_bf16x2(w8[4], w8[5]),
                                     pack_bf16x2(w8[6], w8[7]));
            }
          }
        }
      }
    }
    if (!FOLD) break;
    // end of the pass: every role is done with TMEM, shared memory and the
    // barriers of this pass; run the safe pass if a row asked for it
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (*redo_flag == 0u || *abort_flag != 0u) break;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

template <int DP, int NS, int POLY, int BK, int MINB, bool MASK, bool FOLD>
cudaError_t launch_impl_shape(const AttnLaunch& a, cudaStream_t stream) {
  using Lay = Layout<DP, NS, BK>;
  // key tiles of BK tokens: the query tile's rows (BK == 128), half of them,
  // or half a row when the query tile is a single 128-wide row
  int tck = a.tc, trk = a.tr;
  if (BK == 64) {
    if (a.tr >= 2) trk = a.tr / 2;
    else tck = a.tc / 2;
  }
  CUtensorMap tq, tk, tv, tqp, tkp;
  const int nwx = (a.W + a.M - 1) / a.M, nwy = (a.H + a.M - 1) / a.M;
  const int Hp = nwy * a.M, Wp = nwx * a.M;
  const CUtensorMapSwizzle swc = DP == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  const uint64_t dims5[5] = {uint64_t(DP), uint64_t(a.heads), uint64_t(Wp), uint64_t(Hp), uint64_t(a.B)};
  const uint64_t str5[4] = {uint64_t(DP) * 2, uint64_t(a.heads) * DP * 2, uint64_t(Wp) * a.heads * DP * 2,
                            uint64_t(Hp) * Wp * a.heads * DP * 2};
  const uint32_t box5[5] = {uint32_t(DP), 1u, uint32_t(a.tc), uint32_t(a.tr), 1u};
  const uint32_t box5k[5] = {uint32_t(DP), 1u, uint32_t(tck), uint32_t(trk), 1u};
  const uint64_t dimsv[5] = {32u, uint64_t(a.heads), uint64_t(Wp), uint64_t(Hp), uint64_t(a.B)};
  const uint64_t strv[4] = {64u, uint64_t(a.heads) * 64, uint64_t(Wp) * a.heads * 64, uint64_t(Hp) * Wp * a.heads * 64};
  const uint32_t boxv[5] = {32u, 1u, uint32_t(tck), uint32_t(trk), 1u};
  const uint64_t dims4[4] = {uint64_t(kR), uint64_t(a.M), uint64_t(a.M), uint64_t(a.heads)};
  const uint64_t str4[3] = {uint64_t(kR) * 2, uint64_t(a.M) * kR * 2, uint64_t(a.M) * a.M * kR * 2};
  const uint32_t box4[4] = {uint32_t(kR), uint32_t(a.tc), uint32_t(a.tr), 1u};
  const uint32_t box4k[4] = {uint32_t(kR), uint32_t(tck), uint32_t(trk), 1u};
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (encode_tiled(&tq, bf, 5, const_cast<void*>(a.Qc), dims5, str5, box5, swc) != CUDA_SUCCESS ||
      encode_tiled(&tk, bf, 5, const_cast<void*>(a.Kc), dims5, str5, box5k, swc) != CUDA_SUCCESS ||
      encode_tiled(&tv, bf, 5, const_cast<void*>(a.V), dimsv, strv, boxv, CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS ||
      encode_tiled(&tqp, bf, 4, const_cast<void*>(a.qp), dims4, str4, box4, CU_TENSOR_MAP_SWIZZLE_32B) != CUDA_SUCCESS ||
      encode_tiled(&tkp, bf, 4, const_cast<void*>(a.kp), dims4, str4, box4k, CU_TENSOR_MAP_SWIZZLE_32B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  AttnParams p;
  p.B = a.B; p.H = a.H; p.W = a.W; p.C = a.C; p.heads = a.heads; p.dh = a.dh; p.M = a.M;
  p.tc = a.tc; p.tr = a.tr; p.tiles_x = a.M / a.tc;
  p.n_tiles = (a.M * a.M) / kBQ;
  p.tck = tck;
  p.trk = trk;
  p.tiles_xk = a.M / tck;
  p.n_kv = (a.M * a.M) / BK;
  p.nwx = (a.W + a.M - 1) / a.M;
  p.nwy = (a.H + a.M - 1) / a.M;
  p.Hp = p.nwy * a.M;
  p.Wp = p.nwx * a.M;
  p.scale_log2 = a.scale_log2;
  p.gate = static_cast<const __nv_bfloat16*>(a.gate);
  p.resid = a.resid;
  p.Y = a.Y;
  p.out_f32 = a.out_f32;
  p.out_f16 = a.out_f16;
  p.lse = a.lse;
  p.O_out = static_cast<__nv_bfloat16*>(a.O_out);
  p.err = device_error_word();

  auto kern = rib_attn_fwd_kernel<DP, NS, POLY, BK, MINB, MASK, FOLD>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::ALLOC);
  if (e != cudaSuccess) return e;
  const long long units = static_cast<long long>(a.B) * p.nwy * p.nwx * a.heads * p.n_tiles;
  if (units <= 0) return cudaSuccess;
  kern<<<static_cast<unsigned>(units), kThreads, Lay::ALLOC, stream>>>(tq, tk, tv, tqp, tkp, p);
  return cudaGetLastError();
}

template <int DP, int NS, int POLY, int BK, int MINB>
cudaError_t launch_impl(const AttnLaunch& a, cudaStream_t stream) {
  const bool padded = (a.H % a.M) != 0 || (a.W % a.M) != 0;
  if (a.mask_padding && padded) return launch_impl_shape<DP, NS, POLY, BK, MINB, true, false>(a, stream);
  // the folded softmax needs a spare content column (dh < DP) for the reference
  if (a.dh < DP) return launch_impl_shape<DP, NS, POLY, BK, MINB, false, true>(a, stream);
  return launch_impl_shape<DP, NS, POLY, BK, MINB, false, false>(a, stream);
}

}  // namespace

cudaError_t launch_window_attention(const AttnLaunch& a, cudaStream_t stream) {
  // Block shape (measured on B200): 64-key tiles with four CTAs per SM and 3
  // K/V stages for every head width and window; the 128-key shape with two
  // CTAs per SM was slower at windows 64 and 96 (16-wide heads) and 96
  // (32-wide) once the P.V products went out from their own thread.
  if (a.DP == 32) return launch_impl<32, 3, RIB_ATTN_POLY_SMALL, 64, RIB_ATTN_MINB_SMALL>(a, stream);
  return launch_impl<16, 3, RIB_ATTN_POLY_SMALL, 64, RIB_ATTN_MINB_SMALL>(a, stream);
}

}  // namespace rib
