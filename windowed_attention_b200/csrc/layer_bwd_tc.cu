// Tensor-core backward of the layer's token-wise parts: the content
// projections Qc = q_scale X Wq, Kc = X Wk, V = X Wv ("Résumé technique" 2.A)
// and the CLA pointwise conv G = D Wpw + bpw (RIB/SST write-up section 2.3).
// With g_j the gradients of the projection outputs (fp32, head-padded layout
// [B][Hp][Wp][heads][32]) and dG the gradient of G (bf16 [B][H][W][C]):
//   token GEMMs        dX = sum_j (s_j g_j) W_j^T,       dD = dG Wpw^T
//   token reductions   dW_j = X^T (s_j g_j),             dWpw = D^T dG
// Both run on tcgen05 over tiles of 4 map rows x 32 columns (128 tokens):
//  * fp32 gradients enter the MMA as two bf16 operands, hi = bf16(v) and
//    lo = bf16(v - hi), so each product is exact to about 2^-17 of v (the
//    weights and the bf16 maps are exact in bf16); the tensor core adds in
//    fp32;
//  * the bf16 maps ([T][C] rows, not 16-byte strided when C % 8 != 0) arrive
//    as one bulk copy per map row of the tile and are reformatted in shared
//    memory into 128-byte-swizzled atoms of 64 channels;
//  * the gradients g_j arrive by TMA as boxes of two heads (32 d x 2 heads x
//    32 x 4 rows, fp32, 128-byte swizzle) and are split into the hi/lo atoms;
//  * one atom layout [128 tokens][64 elements] serves as the K-major A
//    operand of the token GEMM (M = tokens) and as the MN-major operands of
//    the token reduction (K = tokens), so no transposes are needed.
// The token GEMM's output leaves by TMA tensor stores (fp32 boxes of 32
// channels, clipped at the map's edges). The token reduction keeps its
// [channels][outputs] accumulator in TMEM over a contiguous range of tiles per
// CTA and writes it once as a partial sum; a second kernel adds the partials
// in chunk order, so the weight gradients are bit-identical from run to run.
//
// Warp roles (512 threads, one CTA per SM):
//   warp 0       producer (one thread: TMA / bulk copies)
//   warp 1       TMEM allocation; one thread issues the MMAs
//   warps 2-11   converters (hi/lo split, map reformat)
//   warps 12-15  epilogue (one TMEM lane quarter each)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "rib_internal.h"
#include "sm100.cuh"

namespace rib {

namespace {

constexpr int kTY = 4, kTX = 32, kRows = kTY * kTX;   // token tile: 4 map rows x 32 columns
constexpr int kAtom = kRows * 128;                    // one atom: 128 rows x 128 bytes (64 bf16)
constexpr int kThreads = 512;
constexpr int kConv0 = 2, kConvWarps = 10, kConvThreads = kConvWarps * 32;
constexpr int kEpi0 = 12;
constexpr int kSmemLimit = 227 * 1024;

enum TcBwdSite : int {
  SITE_T_RAW_FREE = 501, SITE_T_RAW_FULL = 502, SITE_T_A_FREE = 503, SITE_T_A_FULL = 504, SITE_T_W_FREE = 505,
  SITE_T_W_FULL = 506, SITE_T_ACC_FREE = 507, SITE_T_ACC_FULL = 508, SITE_T_DRAIN = 509,
};

struct TcBwdParams {
  int B, H, W, C, heads, dh;
  int ty_n, tx_n;            // tiles per image along y and x
  long long n_tiles;
  int na;                    // g atoms per job: ceil(heads / 2)
  int nc;                    // channel atoms of a map: ceil(C / 64)
  int nk;                    // token GEMM: K atoms per tile (3 na or nc)
  int npad;                  // token GEMM: output columns, a multiple of 32 (MMA N)
  int nacc;                  // token reduction: accumulator columns per 128 channels (64 na or 64 nc)
  int nmh;                   // token reduction: 128-channel halves of the accumulator (1 or 2)
  int hbox;                  // heads per g box (2, or 1 when heads == 1)
  float s[3];                // scale of each job's gradient
  const __nv_bfloat16* mapA; // token GEMM (gate): dG; token reduction: X or D
  const __nv_bfloat16* mapB; // token reduction (gate): dG
  const uint8_t* wimg;       // token GEMM: weight atoms [nk][npad][128 B]
  float* partial;            // token reduction: [chunk][job][C][C]
  int tiles_per_chunk;
  int span;                  // bytes of one map row of a tile in shared memory (32 C 2)
  int raw_slot, nraw;        // raw ring: bytes per slot, slots (token reduction)
  int off_a, off_w, off_st, off_misc;
  int* err;
};

struct TileXY {
  int b, y0, x0;
};
__device__ __forceinline__ TileXY tile_xy(long long tile, int ty_n, int tx_n) {
  TileXY t;
  const long long per_b = static_cast<long long>(ty_n) * tx_n;
  t.b = static_cast<int>(tile / per_b);
  const int r = static_cast<int>(tile - static_cast<long long>(t.b) * per_b);
  t.y0 = (r / tx_n) * kTY;
  t.x0 = (r - (r / tx_n) * tx_n) * kTX;
  return t;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* m, const void* src, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ bool named_all(int id, int n, bool v) {
  uint32_t r;
  asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
               : "=r"(r) : "r"(v ? 1u : 0u), "r"(id), "r"(n) : "memory");
  return r != 0;
}
__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// Producer: one bulk copy per map row of the tile (rows past the map are not
// copied; the reformat writes zeros for them). A row's bytes and source are
// 16-byte multiples when W*C % 8 == 0 and the map is 16-byte aligned.
__device__ __forceinline__ void load_map_tile(uint8_t* dst, const __nv_bfloat16* map, const TileXY& t,
                                              const TcBwdParams& p, uint64_t* bar) {
  const int ntok = p.W - t.x0 < kTX ? p.W - t.x0 : kTX;
  const int rows = p.H - t.y0 < kTY ? p.H - t.y0 : kTY;
  const uint32_t bytes = static_cast<uint32_t>(ntok * p.C * 2);
  mbar_arrive_expect_tx(bar, bytes * rows);
  for (int y = 0; y < rows; ++y)
    bulk_load(dst + y * p.span, map + ((static_cast<size_t>(t.b) * p.H + t.y0 + y) * p.W + t.x0) * p.C, bytes, bar);
}

// Converter: channel atom `a` (channels 64a .. 64a+63) of a raw map tile ->
// [128 rows][128 B] with the 16-byte chunks of row r permuted by r % 8
// (tcgen05's 128-byte swizzle); row r = 32 y + x; zeros past the map and
// past C.
__device__ __forceinline__ void reformat_atom(uint8_t* atom, int a, const uint8_t* raw, const TileXY& t,
                                              const TcBwdParams& p, int tid, int nthr) {
  const int ntok = p.W - t.x0 < kTX ? p.W - t.x0 : kTX;
  const int rows = p.H - t.y0 < kTY ? p.H - t.y0 : kTY;
  const int cq = p.C / 4;
  for (int i = tid; i < kRows * 16; i += nthr) {
    const int r = i >> 4, q = i & 15;           // row, 8-byte piece (4 channels) of the atom
    const int y = r >> 5, x = r & 31, pc = 16 * a + q;
    uint2 v = make_uint2(0u, 0u);
    if (y < rows && x < ntok && pc < cq) v = *reinterpret_cast<const uint2*>(raw + y * p.span + (x * p.C + 4 * pc) * 2);
    *reinterpret_cast<uint2*>(atom + r * 128 + ((((q >> 1) ^ (r & 7))) << 4) + (q & 1) * 8) = v;
  }
}

// Converter: raw g box (TMA, 128-byte swizzle: 128-byte segment sg = 2 r + h
// holds d = 0..31 of head h of row r, its 16-byte chunk c at sg*128 +
// ((c ^ (sg % 8)) * 16)) -> hi and lo atoms, element (r, 32 h + d) = s * g.
__device__ __forceinline__ void convert_g_atom(uint8_t* hi, uint8_t* lo, const uint8_t* raw, float s, int hbox,
                                               int tid, int nthr) {
  for (int i = tid; i < kRows * 16; i += nthr) {
    const int c = i & 7, sg = i >> 3, r = sg >> 1, h = sg & 1;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (h < hbox) v = *reinterpret_cast<const float4*>(raw + (r * hbox + h) * 128 + ((c ^ ((r * hbox + h) & 7)) << 4));
    const float f0 = v.x * s, f1 = v.y * s, f2 = v.z * s, f3 = v.w * s;
    const uint32_t h01 = pack_bf16x2(f0, f1), h23 = pack_bf16x2(f2, f3);
    const uint32_t l01 = pack_bf16x2(f0 - bf16_lo(h01), f1 - bf16_hi(h01));
    const uint32_t l23 = pack_bf16x2(f2 - bf16_lo(h23), f3 - bf16_hi(h23));
    // elements 32 h + 4 c .. +3: 16-byte chunk 4 h + c / 2, half c % 2
    const uint32_t off = r * 128 + ((((4 * h + (c >> 1)) ^ (r & 7))) << 4) + (c & 1) * 8;
    *reinterpret_cast<uint2*>(hi + off) = make_uint2(h01, h23);
    *reinterpret_cast<uint2*>(lo + off) = make_uint2(l01, l23);
  }
}

// ---------------------------------------------------------------------------
// Token GEMM: out[t][n] = sum_k A[t][k] Wimg[k][n], fp32, over tiles of 128
// tokens. MODE 0: A = (s_j g_j) for the three jobs, K atoms (job, 2 heads),
// hi and lo MMAs per atom; out = dX. MODE 1: A = dG (map), K atoms of 64
// channels; out = dD. The weight atoms stream through a two-slot ring (they
// are re-read from L2 for every tile).
// ---------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_gemm_kernel(const __grid_constant__ CUtensorMap g0, const __grid_constant__ CUtensorMap g1,
                   const __grid_constant__ CUtensorMap g2, const __grid_constant__ CUtensorMap out_map,
                   const TcBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* sRaw = smem;                  // MODE 0: two 32 KB g boxes; MODE 1: one map tile
  uint8_t* sA = smem + p.off_a;          // two 32 KB slots (MODE 0: hi | lo atom; MODE 1: one atom)
  uint8_t* sW = smem + p.off_w;          // two weight slots of npad * 128 bytes
  uint8_t* sSt = smem + p.off_st;        // two 16 KB store boxes
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_misc);
  uint64_t* raw_full = bars;        // [2]
  uint64_t* raw_free = bars + 2;    // [2]
  uint64_t* a_full = bars + 4;      // [2]
  uint64_t* a_free = bars + 6;      // [2]
  uint64_t* w_full = bars + 8;      // [2]
  uint64_t* w_free = bars + 10;     // [2]
  uint64_t* acc_full = bars + 12;   // [2]
  uint64_t* acc_free = bars + 14;   // [2]
  uint64_t* done = bars + 16;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 17);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(tmem_holder + 1);
  const int wslot = p.npad * 128;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_free[i], kConvWarps);
      mbar_init(&a_full[i], kConvWarps);
      mbar_init(&a_free[i], 1);
      mbar_init(&w_full[i], 1);
      mbar_init(&w_free[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_free[i], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0u;
    tmem_holder[2] = 0u;   // abort word of the teardown drains (never raised)
    fence_barrier_init();
    if (MODE == 0) {
      tma_prefetch_desc(&g0);
      tma_prefetch_desc(&g1);
      tma_prefetch_desc(&g2);
    }
    tma_prefetch_desc(&out_map);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, p.err};
  const WaitCtx drain{reinterpret_cast<volatile uint32_t*>(tmem_holder + 2), p.err};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int q = 0, qg = 0, last_tile = -1;   // q: weight atoms issued, qg: g boxes issued
      long long tc = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++tc) {
        const TileXY t = tile_xy(tile, p.ty_n, p.tx_n);
        if (MODE == 1) {
          if (tc >= 1 && !(ok = mbar_wait(&raw_free[0], (tc - 1) & 1, wc, SITE_T_RAW_FREE))) break;
          load_map_tile(sRaw, p.mapA, t, p, &raw_full[0]);
          last_tile = static_cast<int>(tc);
        }
        for (int k = 0; k < p.nk; ++k, ++q) {
          const int s = q & 1;
          if (MODE == 0) {
            if (q >= 2 && !(ok = mbar_wait(&raw_free[s], ((q >> 1) - 1) & 1, wc, SITE_T_RAW_FREE))) break;
            const int j = k / p.na, a = k - j * p.na;
            mbar_arrive_expect_tx(&raw_full[s], static_cast<uint32_t>(kRows * p.hbox * 128));
            tma_load_5d(sRaw + s * 2 * kAtom, j == 0 ? &g0 : (j == 1 ? &g1 : &g2), &raw_full[s], 0, 2 * a, t.x0, t.y0,
                        t.b);
            ++qg;
          }
          if (q >= 2 && !(ok = mbar_wait(&w_free[s], ((q >> 1) - 1) & 1, wc, SITE_T_W_FREE))) break;
          mbar_arrive_expect_tx(&w_full[s], static_cast<uint32_t>(wslot));
          bulk_load(sW + s * wslot, p.wimg + static_cast<size_t>(k) * wslot, static_cast<uint32_t>(wslot), &w_full[s]);
        }
      }
      // drain: every copy issued has landed before the CTA may exit
      for (int i = qg - 2 > 0 ? qg - 2 : 0; i < qg; ++i) mbar_wait(&raw_full[i & 1], (i >> 1) & 1, drain, SITE_T_DRAIN);
      for (int i = q - 2 > 0 ? q - 2 : 0; i < q; ++i) mbar_wait(&w_full[i & 1], (i >> 1) & 1, drain, SITE_T_DRAIN);
      if (MODE == 1 && last_tile >= 0) mbar_wait(&raw_full[0], last_tile & 1, drain, SITE_T_DRAIN);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, p.npad, false, false);
      int q = 0, it = 0;
      bool ok = true;
      for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++it) {
        const int ab = it & 1;
        if (it >= 2 && !(ok = mbar_wait(&acc_free[ab], ((it >> 1) - 1) & 1, wc, SITE_T_ACC_FREE))) break;
        tc_fence_after();
        const uint32_t acc = tmem + 256u * ab;
        for (int k = 0; k < p.nk; ++k, ++q) {
          const int s = q & 1;
          if (!(ok = mbar_wait(&a_full[s], (q >> 1) & 1, wc, SITE_T_A_FULL))) break;
          if (!(ok = mbar_wait(&w_full[s], (q >> 1) & 1, wc, SITE_T_W_FULL))) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * 2 * kAtom), w0 = smem_u32(sW + s * wslot);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            // K step ks: 32-byte offset inside the 128-byte rows
            const uint64_t bd = make_sdesc(w0 + 32 * ks, 16, 1024, SW_128B);
            umma_ss(acc, make_sdesc(a0 + 32 * ks, 16, 1024, SW_128B), bd, idesc, (k > 0 || ks > 0) ? 1u : 0u);
            if (MODE == 0) umma_ss(acc, make_sdesc(a0 + kAtom + 32 * ks, 16, 1024, SW_128B), bd, idesc, 1u);
          }
          umma_commit(&a_free[s]);
          umma_commit(&w_free[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
      }
      umma_commit(done);
      mbar_wait(done, 0, drain, SITE_T_DRAIN);
    }
  } else if (warp < kEpi0) {
    // ------------------------------------------------------------ converters
    const int ct = tid - kConv0 * 32;
    int q = 0;
    long long tc = 0;
    bool ok = true;
    for (long long tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++tc) {
      const TileXY t = tile_xy(tile, p.ty_n, p.tx_n);
      if (MODE == 1 && !(ok = warp_all(mbar_wait(&raw_full[0], tc & 1, wc, SITE_T_RAW_FULL)))) break;
      for (int k = 0; k < p.nk; ++k, ++q) {
        const int s = q & 1;
        if (MODE == 0 && !(ok = warp_all(mbar_wait(&raw_full[s], (q >> 1) & 1, wc, SITE_T_RAW_FULL)))) break;
        if (q >= 2 && !(ok = warp_all(mbar_wait(&a_free[s], ((q >> 1) - 1) & 1, wc, SITE_T_A_FREE)))) break;
        uint8_t* a = sA + s * 2 * kAtom;
        if (MODE == 0) {
          const int j = k / p.na;
          convert_g_atom(a, a + kAtom, sRaw + s * 2 * kAtom, j == 0 ? p.s[0] : (j == 1 ? p.s[1] : p.s[2]), p.hbox, ct,
                         kConvThreads);
        } else {
          reformat_atom(a, k, sRaw, t, p, ct, kConvThreads);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&a_full[s]);
          if (MODE == 0) mbar_arrive(&raw_free[s]);
        }
      }
      if (!ok) break;
      if (MODE == 1) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_free[0]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const bool leader = warp == kEpi0 && lane == 0;
    int it = 0, box = 0;
    for (long long tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++it) {
      const int ab = it & 1;
      const bool ok = named_all(1, 128, mbar_wait(&acc_full[ab], (it >> 1) & 1, wc, SITE_T_ACC_FULL));
      if (!ok) break;
      tc_fence_after();
      const TileXY t = tile_xy(tile, p.ty_n, p.tx_n);
      const uint32_t acc = tmem + 256u * ab + lane_off;
      for (int cb = 0; cb < p.npad / 32; ++cb, ++box) {
        uint32_t v[32];
        tmem_ld32(acc + 32 * cb, v);
        tmem_wait_ld();
        uint8_t* sb = sSt + (box & 1) * kAtom;
        if (leader) bulk_wait_read1();   // the store issued from this buffer two boxes ago has read it
        named_sync(1, 128);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(sb + row * 128 + ((c ^ (row & 7)) << 4)) =
              make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        fence_proxy_async_smem();
        named_sync(1, 128);
        if (leader) {
          tma_store_4d(&out_map, sb, 32 * cb, t.x0, t.y0, t.b);
          bulk_commit();
        }
      }
      // accumulator drained: the MMAs of tile it + 2 may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_free[ab]);
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

// ---------------------------------------------------------------------------
// Token reduction: partial[chunk][job][c][n] = sum over this CTA's tiles of
// A[t][c] Bop[t][n], A = X (MODE 0) or D (MODE 1) from the map, Bop = s_j g_j
// (MODE 0, hi and lo, job = blockIdx.y) or dG (MODE 1). The accumulator
// [128 channels x nacc] x nmh lives in TMEM for the whole tile range; MMAs of
// N = 64 per B atom, both operands MN-major (K = tokens).
// ---------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_wgrad_kernel(const __grid_constant__ CUtensorMap g0, const __grid_constant__ CUtensorMap g1,
                    const __grid_constant__ CUtensorMap g2, const TcBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* sRaw = smem;                  // nraw slots of raw_slot bytes
  uint8_t* sX = smem + p.off_a;          // nc channel atoms of A (an atom past them is read as padding)
  uint8_t* sB = smem + p.off_w;          // MODE 0: two 32 KB hi|lo slots; MODE 1: nc atoms of dG
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_misc);
  uint64_t* raw_full = bars;        // [2]
  uint64_t* raw_free = bars + 2;    // [2]
  uint64_t* x_full = bars + 4;
  uint64_t* x_free = bars + 5;
  uint64_t* b_full = bars + 6;      // [2]
  uint64_t* b_free = bars + 8;      // [2]
  uint64_t* acc_full = bars + 10;
  uint64_t* done = bars + 11;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 12);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(tmem_holder + 1);
  const int job = MODE == 0 ? blockIdx.y : 0;
  const long long tb = static_cast<long long>(blockIdx.x) * p.tiles_per_chunk;
  const long long te = tb + p.tiles_per_chunk < p.n_tiles ? tb + p.tiles_per_chunk : p.n_tiles;
  const int items = MODE == 0 ? 1 + p.na : 2;   // raw items per tile: the A map, then B's pieces

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_free[i], kConvWarps);
      mbar_init(&b_full[i], kConvWarps);
      mbar_init(&b_free[i], 1);
    }
    mbar_init(x_full, kConvWarps);
    mbar_init(x_free, 1);
    mbar_init(acc_full, 1);
    mbar_init(done, 1);
    *abort_flag = 0u;
    tmem_holder[2] = 0u;
    fence_barrier_init();
    if (MODE == 0) tma_prefetch_desc(job == 0 ? &g0 : (job == 1 ? &g1 : &g2));
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, p.err};
  const WaitCtx drain{reinterpret_cast<volatile uint32_t*>(tmem_holder + 2), p.err};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int r = 0;   // raw items issued
      bool ok = true;
      const CUtensorMap* gm = job == 0 ? &g0 : (job == 1 ? &g1 : &g2);
      for (long long tile = tb; tile < te && ok; ++tile) {
        const TileXY t = tile_xy(tile, p.ty_n, p.tx_n);
        for (int k = 0; k < items; ++k, ++r) {
          const int s = r % p.nraw, use = r / p.nraw;
          if (use >= 1 && !(ok = mbar_wait(&raw_free[s], (use - 1) & 1, wc, SITE_T_RAW_FREE))) break;
          uint8_t* dst = sRaw + s * p.raw_slot;
          if (k == 0) {
            load_map_tile(dst, p.mapA, t, p, &raw_full[s]);
          } else if (MODE == 1) {
            load_map_tile(dst, p.mapB, t, p, &raw_full[s]);
          } else {
            mbar_arrive_expect_tx(&raw_full[s], static_cast<uint32_t>(kRows * p.hbox * 128));
            tma_load_5d(dst, gm, &raw_full[s], 0, 2 * (k - 1), t.x0, t.y0, t.b);
          }
        }
      }
      for (int i = r - p.nraw > 0 ? r - p.nraw : 0; i < r; ++i)
        mbar_wait(&raw_full[i % p.nraw], (i / p.nraw) & 1, drain, SITE_T_DRAIN);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, 64, true, true);
      const uint32_t x0 = smem_u32(sX);
      int qb = 0, n = 0;
      bool ok = true;
      for (long long tile = tb; tile < te && ok; ++tile, ++n) {
        if (!(ok = mbar_wait(x_full, n & 1, wc, SITE_T_A_FULL))) break;
        const int nb = MODE == 0 ? p.na : 1;   // B hand-offs per tile
        for (int k = 0; k < nb; ++k, ++qb) {
          const int s = MODE == 0 ? (qb & 1) : 0;
          const uint32_t ph = MODE == 0 ? ((qb >> 1) & 1) : (qb & 1);
          if (!(ok = mbar_wait(&b_full[s], ph, wc, SITE_T_W_FULL))) break;
          tc_fence_after();
          const int a_lo = MODE == 0 ? k : 0, a_hi = MODE == 0 ? k + 1 : p.nc;
          for (int a = a_lo; a < a_hi; ++a) {
            // B atom: MODE 0 the hi|lo pair of this g atom, MODE 1 dG channel atom a
            const uint32_t b0 = MODE == 0 ? smem_u32(sB + s * 2 * kAtom) : smem_u32(sB + a * kAtom);
            for (int mh = 0; mh < p.nmh; ++mh) {
              const uint32_t acc = tmem + static_cast<uint32_t>(mh * p.nacc + 64 * a);
#pragma unroll 2
              for (int ks = 0; ks < kRows / 16; ++ks) {
                // K step ks = 16 tokens = two 8-row groups (SBO 1024); the
                // 128 channels of half mh are two atoms (LBO one atom)
                const uint64_t ad = make_sdesc(x0 + 2 * mh * kAtom + 2048 * ks, kAtom, 1024, SW_128B);
                const uint32_t en = (n > 0 || ks > 0) ? 1u : 0u;
                umma_ss(acc, ad, make_sdesc(b0 + 2048 * ks, kAtom, 1024, SW_128B), idesc, en);
                if (MODE == 0) umma_ss(acc, ad, make_sdesc(b0 + kAtom + 2048 * ks, kAtom, 1024, SW_128B), idesc, 1u);
              }
            }
          }
          umma_commit(&b_free[s]);
        }
        if (!ok) break;
        umma_commit(x_free);
      }
      umma_commit(acc_full);
      umma_commit(done);
      mbar_wait(done, 0, drain, SITE_T_DRAIN);
    }
  } else if (warp < kEpi0) {
    // ------------------------------------------------------------ converters
    const int ct = tid - kConv0 * 32;
    int r = 0, qb = 0, n = 0;
    bool ok = true;
    for (long long tile = tb; tile < te && ok; ++tile, ++n) {
      const TileXY t = tile_xy(tile, p.ty_n, p.tx_n);
      for (int k = 0; k < items; ++k, ++r) {
        const int s = r % p.nraw, use = r / p.nraw;
        if (!(ok = warp_all(mbar_wait(&raw_full[s], use & 1, wc, SITE_T_RAW_FULL)))) break;
        const uint8_t* raw = sRaw + s * p.raw_slot;
        if (k == 0) {
          // A atoms: the MMAs of the previous tile have read them
          if (n >= 1 && !(ok = warp_all(mbar_wait(x_free, (n - 1) & 1, wc, SITE_T_A_FREE)))) break;
          for (int a = 0; a < p.nc; ++a) reformat_atom(sX + a * kAtom, a, raw, t, p, ct, kConvThreads);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(x_full);
            mbar_arrive(&raw_free[s]);
          }
        } else {
          const int bs = MODE == 0 ? (qb & 1) : 0;
          const int bu = MODE == 0 ? (qb >> 1) : qb;
          if (bu >= 1 && !(ok = warp_all(mbar_wait(&b_free[bs], (bu - 1) & 1, wc, SITE_T_W_FREE)))) break;
          if (MODE == 0) {
            uint8_t* b = sB + bs * 2 * kAtom;
            convert_g_atom(b, b + kAtom, raw, job == 0 ? p.s[0] : (job == 1 ? p.s[1] : p.s[2]), p.hbox, ct,
                           kConvThreads);
          } else {
            for (int a = 0; a < p.nc; ++a) reformat_atom(sB + a * kAtom, a, raw, t, p, ct, kConvThreads);
          }
          ++qb;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&b_full[bs]);
            mbar_arrive(&raw_free[s]);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const bool ok = named_all(1, 128, mbar_wait(acc_full, 0, wc, SITE_T_ACC_FULL));
    if (ok && te > tb) {
      tc_fence_after();
      const int C = p.C;
      float* out = p.partial + (static_cast<size_t>(blockIdx.x) * gridDim.y + job) * C * C;
      for (int mh = 0; mh < p.nmh; ++mh) {
        const int c = 128 * mh + quarter * 32 + lane;   // input channel = accumulator row
        for (int g32 = 0; g32 < p.nacc / 32; ++g32) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + static_cast<uint32_t>(mh * p.nacc + 32 * g32), v);
          tmem_wait_ld();
          if (c >= C) continue;
          float* orow = out + static_cast<size_t>(c) * C;
          if (MODE == 0) {
            // accumulator column 32 h + d is output column h dh + d (d < dh)
            if (g32 < p.heads) {
#pragma unroll
              for (int d = 0; d < 32; ++d)
                if (d < p.dh) orow[g32 * p.dh + d] = __uint_as_float(v[d]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (32 * g32 + e < C) orow[32 * g32 + e] = __uint_as_float(v[e]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Weight atoms of the token GEMM, [nk][npad rows][128 B] in the 128-byte
// swizzled K-major layout: row n (output channel), element k of atom kk.
//  MODE 0: atom kk = (job j, heads 2a, 2a+1), k = 32 h + d -> W_j[n][(2a+h) dh + d]
//          (zero for d >= dh, heads past the last, n >= C);
//  MODE 1: atom kk = channels 64 kk .., k -> Wpw[n][64 kk + k] (zero past C).
__global__ void tc_bwd_weight_image_kernel(const __nv_bfloat16* __restrict__ W0, const __nv_bfloat16* __restrict__ W1,
                                           const __nv_bfloat16* __restrict__ W2, uint8_t* __restrict__ img, int mode,
                                           int nk, int na, int npad, int C, int heads, int dh) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;   // one 16-byte chunk: (kk, n, chunk)
  if (i >= nk * npad * 8) return;
  const int ch = i & 7, n = (i >> 3) % npad, kk = (i >> 3) / npad;
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint32_t two = 0;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int k = 8 * ch + 2 * e + u;
      uint16_t bits = 0;
      if (n < C) {
        if (mode == 0) {
          const int j = kk / na, a = kk - j * na, h = 2 * a + (k >> 5), d = k & 31;
          const __nv_bfloat16* Wj = j == 0 ? W0 : (j == 1 ? W1 : W2);
          if (h < heads && d < dh) bits = __bfloat16_as_ushort(Wj[static_cast<size_t>(n) * C + h * dh + d]);
        } else {
          const int m = 64 * kk + k;
          if (m < C) bits = __bfloat16_as_ushort(W0[static_cast<size_t>(n) * C + m]);
        }
      }
      two |= static_cast<uint32_t>(bits) << (16 * u);
    }
    w[e] = two;
  }
  *reinterpret_cast<uint4*>(img + static_cast<size_t>(kk) * npad * 128 + n * 128 + ((ch ^ (n & 7)) << 4)) =
      make_uint4(w[0], w[1], w[2], w[3]);
}

// Partial sums of the weight gradients in chunk order:
// out_j[i] = sum_k partial[(k * jobs + j) * n + i], i < n.
__global__ void wgrad_partial_sum_kernel(const float* __restrict__ partial, int chunks, int jobs, int n,
                                         float* __restrict__ o0, float* __restrict__ o1, float* __restrict__ o2) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int j = blockIdx.y;
  if (i >= n) return;
  float s = 0.f;
  for (int k = 0; k < chunks; ++k) s += partial[(static_cast<size_t>(k) * jobs + j) * n + i];
  (j == 0 ? o0 : (j == 1 ? o1 : o2))[i] = s;
}

}  // namespace

cudaError_t launch_wgrad_partial_sum(const float* partial, int chunks, int jobs, int n, float* o0, float* o1,
                                     float* o2, cudaStream_t stream) {
  if (chunks <= 0 || n <= 0) return cudaSuccess;
  wgrad_partial_sum_kernel<<<dim3((n + 255) / 256, jobs), 256, 0, stream>>>(partial, chunks, jobs, n, o0, o1, o2);
  return cudaGetLastError();
}

bool tc_bwd_supported(const void* map, int H, int W, int C) {
  return map && (reinterpret_cast<uintptr_t>(map) % 16) == 0 && (static_cast<long long>(W) * C) % 8 == 0 &&
         C % 4 == 0 && C >= 32 && C <= 256 && W >= kTX && H >= kTY;
}

size_t tc_bwd_weight_image_bytes(int C, int heads, bool projection) {
  const int npad = (C + 31) / 32 * 32;
  const int nk = projection ? 3 * ((heads + 1) / 2) : (C + 63) / 64;
  return static_cast<size_t>(nk) * npad * 128;
}

size_t wgrad_partial_bytes(int C) { return static_cast<size_t>(kWgradChunks) * C * C * sizeof(float); }

namespace {

TcBwdParams base_params(int B, int H, int W, int C, int heads) {
  TcBwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = B;
  p.H = H;
  p.W = W;
  p.C = C;
  p.heads = heads;
  p.dh = C / heads;
  p.ty_n = (H + kTY - 1) / kTY;
  p.tx_n = (W + kTX - 1) / kTX;
  p.n_tiles = static_cast<long long>(B) * p.ty_n * p.tx_n;
  p.na = (heads + 1) / 2;
  p.nc = (C + 63) / 64;
  p.npad = (C + 31) / 32 * 32;
  p.hbox = heads >= 2 ? 2 : 1;
  p.span = kTX * C * 2;
  p.err = device_error_word();
  return p;
}

CUresult encode_g_map(CUtensorMap* m, const float* g, int B, int Hp, int Wp, int heads, int hbox) {
  const uint64_t dims[5] = {32, uint64_t(heads), uint64_t(Wp), uint64_t(Hp), uint64_t(B)};
  const uint64_t strides[4] = {128, uint64_t(heads) * 128, uint64_t(Wp) * heads * 128,
                               uint64_t(Hp) * Wp * heads * 128};
  const uint32_t box[5] = {32, uint32_t(hbox), uint32_t(kTX), uint32_t(kTY), 1};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, const_cast<float*>(g), dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

CUresult encode_out_map(CUtensorMap* m, float* out, int B, int H, int W, int C) {
  const uint64_t dims[4] = {uint64_t(C), uint64_t(W), uint64_t(H), uint64_t(B)};
  const uint64_t strides[3] = {uint64_t(C) * 4, uint64_t(W) * C * 4, uint64_t(H) * W * C * 4};
  const uint32_t box[4] = {32, uint32_t(kTX), uint32_t(kTY), 1};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, out, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

cudaError_t launch_gemm(int mode, TcBwdParams p, const CUtensorMap* g, const CUtensorMap& out_map,
                        cudaStream_t stream) {
  p.nk = mode == 0 ? 3 * p.na : p.nc;
  p.off_a = 2 * 2 * kAtom;                       // raw: two g boxes or one map tile (<= 64 KB)
  p.off_w = p.off_a + 2 * 2 * kAtom;
  p.off_st = p.off_w + 2 * p.npad * 128;
  p.off_misc = p.off_st + 2 * kAtom;
  const int total = p.off_misc + 256 + 1024;
  if (total > kSmemLimit) return cudaErrorInvalidConfiguration;
  if (p.n_tiles == 0) return cudaSuccess;
  auto kern = mode == 0 ? tc_bwd_gemm_kernel<0> : tc_bwd_gemm_kernel<1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, total);
  if (e != cudaSuccess) return e;
  const long long grid = p.n_tiles < sm_count() ? p.n_tiles : sm_count();
  kern<<<static_cast<unsigned>(grid), kThreads, total, stream>>>(g[0], g[1], g[2], out_map, p);
  return cudaGetLastError();
}

cudaError_t launch_wgrad(int mode, TcBwdParams p, const CUtensorMap* g, int* chunks_out, cudaStream_t stream) {
  const int jobs = mode == 0 ? 3 : 1;
  const int per_job = kWgradChunks / jobs;
  long long tpc = (p.n_tiles + per_job - 1) / per_job;
  if (tpc < 1) tpc = 1;
  const int chunks = static_cast<int>((p.n_tiles + tpc - 1) / tpc);
  p.tiles_per_chunk = static_cast<int>(tpc);
  p.nacc = mode == 0 ? 64 * p.na : 64 * p.nc;
  p.nmh = p.C > 128 ? 2 : 1;
  const int map_bytes = kTY * p.span;
  p.raw_slot = (mode == 0 ? (map_bytes > 2 * kAtom ? map_bytes : 2 * kAtom) : map_bytes);
  p.raw_slot = (p.raw_slot + 1023) / 1024 * 1024;
  const int b_bytes = mode == 0 ? 2 * 2 * kAtom : p.nc * kAtom;
  // the A operand of the upper channel half reads (as padding rows) up to
  // four atoms from sX: keep them inside the allocation
  const int x_bytes = p.nc * kAtom;
  const int x_reach = p.nmh * 2 * kAtom;
  auto layout = [&](int nraw) {
    p.nraw = nraw;
    p.off_a = nraw * p.raw_slot;
    p.off_w = p.off_a + x_bytes;
    p.off_misc = p.off_w + b_bytes;
    int end = p.off_misc + 256;
    if (p.off_a + x_reach > end) end = p.off_a + x_reach;
    return end + 1024;
  };
  int total = layout(2);
  if (total > kSmemLimit) total = layout(1);
  if (total > kSmemLimit) return cudaErrorInvalidConfiguration;
  *chunks_out = chunks;
  if (p.n_tiles == 0) return cudaSuccess;
  auto kern = mode == 0 ? tc_bwd_wgrad_kernel<0> : tc_bwd_wgrad_kernel<1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, total);
  if (e != cudaSuccess) return e;
  dim3 grid(chunks, jobs);
  kern<<<grid, kThreads, total, stream>>>(g[0], g[1], g[2], p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qkv_project_bwd_tc(const QkvBwdLaunch& a, void* ws, cudaStream_t stream) {
  TcBwdParams p = base_params(a.B, a.H, a.W, a.C, a.heads);
  for (int j = 0; j < 3; ++j) p.s[j] = a.s[j];
  p.mapA = static_cast<const __nv_bfloat16*>(a.X);
  uint8_t* img = static_cast<uint8_t*>(ws);
  float* partial = reinterpret_cast<float*>(img + align256(tc_bwd_weight_image_bytes(a.C, a.heads, true)));
  p.wimg = img;
  p.partial = partial;
  const int nk = 3 * p.na;
  const int chunks16 = nk * p.npad * 8;
  tc_bwd_weight_image_kernel<<<(chunks16 + 255) / 256, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(a.Wt[0]), static_cast<const __nv_bfloat16*>(a.Wt[1]),
      static_cast<const __nv_bfloat16*>(a.Wt[2]), img, 0, nk, p.na, p.npad, a.C, a.heads, p.dh);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap g[3], out_map;
  std::memset(g, 0, sizeof(g));
  for (int j = 0; j < 3; ++j)
    if (encode_g_map(&g[j], a.g[j], a.B, a.Hp, a.Wp, a.heads, p.hbox) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_out_map(&out_map, a.dX, a.B, a.H, a.W, a.C) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  e = launch_gemm(0, p, g, out_map, stream);
  if (e != cudaSuccess) return e;
  int chunks = 0;
  e = launch_wgrad(0, p, g, &chunks, stream);
  if (e != cudaSuccess || chunks == 0) return e;
  return launch_wgrad_partial_sum(partial, chunks, 3, a.C * a.C, a.dW[0], a.dW[1], a.dW[2], stream);
}

cudaError_t launch_gate_bwd_tc_gemms(const GateBwdLaunch& a, uint8_t* img, float* partial, cudaStream_t stream,
                                     int* chunks_out) {
  TcBwdParams p = base_params(a.B, a.H, a.W, a.C, 1);
  p.s[0] = p.s[1] = p.s[2] = 1.f;
  p.wimg = img;
  p.partial = partial;
  const int chunks16 = p.nc * p.npad * 8;
  tc_bwd_weight_image_kernel<<<(chunks16 + 255) / 256, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(a.Wpw), nullptr, nullptr, img, 1, p.nc, p.na, p.npad, a.C, 1, a.C);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap g[3], out_map;
  std::memset(g, 0, sizeof(g));
  if (encode_out_map(&out_map, a.dD, a.B, a.H, a.W, a.C) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  // dD = dG Wpw^T
  p.mapA = static_cast<const __nv_bfloat16*>(a.dG);
  e = launch_gemm(1, p, g, out_map, stream);
  if (e != cudaSuccess) return e;
  // dWpw partials = D^T dG
  p.mapA = static_cast<const __nv_bfloat16*>(a.D);
  p.mapB = static_cast<const __nv_bfloat16*>(a.dG);
  return launch_wgrad(1, p, g, chunks_out, stream);
}

}  // namespace rib
