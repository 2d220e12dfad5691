// Token GEMM on tcgen05: out[t, n] = epilogue( sum_k A[t, k] * W'[k, n] ).
//
// Used for two rows of the hot path:
//  * the content projections Qc = X Wq, Kc = X Wk, V = X Wv (the write-up
//    takes these pixel content features as given; "Résumé technique" 2.A),
//    written in the head-padded layout [T][heads][DP] the attention kernel
//    loads with TMA (column n = head*DP + d maps to weight column head*dh + d
//    for d < dh and to a zero column otherwise);
//  * the CLA pointwise conv G = D Wpw + bpw followed by the sigmoid of the
//    gate (RIB/SST write-up section 2.3), written as bf16 [T][C] (the
//    two-pass gate, for maps the fused gate kernel does not take);
//  * the ConvFFN's first linear map with bias and GELU (section 3.1), written
//    as bf16 [T][hidden padded to 8].
//
// Both are HBM-bound (C/2 flop per byte with C <= 256). The kernel is a
// persistent, warp-specialised pipeline, one CTA per SM and one job (one
// weight) per CTA group, so every stage of consecutive 128-token tiles runs
// concurrently:
//   warp 0    producer: maps the output rows of each quarter tile (32 rows)
//             to source rows of A and bulk-copies each run of rows that is
//             contiguous in A (one cp.async.bulk per run, usually one per
//             quarter tile) into a ring of raw stages (four to eight, as many
//             as shared memory holds), so the next rows are in flight while
//             these are reformatted. When a whole tile is one run of rows that
//             meets the bulk copy's 16-byte rules (a tile with no padded token,
//             in the common case), one thread issues its four copies and the
//             reformat warps compute the raw offsets: the per-row tables and
//             warp collectives of the general path cost about a thousand
//             cycles per stage, more than the tile's MMAs.
//             Channels-last rows of C bf16 are only 8-byte aligned when
//             C % 8 != 0, which rules out TMA tensor tiles for A; a run's
//             first or last row that breaks the bulk copy's 16-byte rule is
//             read from global memory by the next stage instead.
//   warps 2-5 reformat the raw rows into the A operand, which lives in
//             TMEM (row = lane, K in columns of bf16 pairs, as tcgen05.mma
//             reads A from tensor memory): warp w serves lane quarter w % 4,
//             i.e. raw stage w % 4 of each tile, thread = row, writing the two
//             K halves in turn.
//             Keeping A out of shared memory leaves room for a raw ring of at
//             least one whole tile (4 to 8 stages), which the bulk copies'
//             latency needs; the two K halves have their own barriers, so the
//             first half of tile i + 1 is written while the MMAs of tile i's
//             second half run.
//   warp 1    one thread issues the K/16 tcgen05.mma of a tile (A from TMEM,
//             W' from shared memory) into one of two TMEM accumulators (one
//             when two do not fit beside A); W' is staged once per CTA in the
//             UMMA K-major 128-byte-swizzled layout, by the epilogue warps
//             while the first tiles load.
//   warps 6-17 epilogue in three groups of four warps (thread = token row, the
//             groups take every third column box; with two groups the
//             epilogue bound the tile rate): TMEM -> registers -> shared
//             staging -> asynchronous stores: TMA tensor stores of swizzled
//             column boxes for the head-padded projection outputs (one or two
//             staging buffers per group), one bulk copy of the contiguous
//             [128][C] rows for the gate.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "rib_internal.h"
#include "sm100.cuh"

namespace rib {

namespace {

constexpr int kTile = 128;
constexpr int kSR = 32;             // rows per raw stage (a quarter tile)
constexpr int kMaxRaw = 8;          // raw stages at most
constexpr int kThreads = 576;       // 18 warps
constexpr int kRefWarps = 4;        // reformat warps (2 .. 5), one per TMEM lane quarter
constexpr int kEpi0 = 2 + kRefWarps; // first epilogue warp
constexpr int kEpiGroups = 3;       // epilogue groups of four warps (one per lane quarter)
constexpr int kEpiThreads = kEpiGroups * 128;
// dynamic shared memory at most: 227 KB less the static arrays (bias, run tables)
constexpr int kSmemLimit = 227 * 1024 - 5120;

enum GemmSite : int {
  SITE_G_RAW_FREE = 201, SITE_G_RAW_FULL = 202, SITE_G_A_FREE = 203, SITE_G_A_FULL = 204,
  SITE_G_ACC_FREE = 205, SITE_G_ACC_FULL = 206, SITE_G_DRAIN = 207, SITE_G_W_READY = 208,
};

struct GemmParams {
  const __nv_bfloat16* A;
  long long T;        // output rows (mode 0: B*Hp*Wp padded-image tokens)
  int B, H, W, Hp, Wp;
  int K, KP, mode, heads, dh, n_real, w_cols;
  int n_valid;        // mode 1: columns with weights and bias (the rest of n_real are zero)
  int a_f16;          // A is fp16: the weights are staged as fp16 and the product runs in fp16
  int gelu;           // mode 1: GELU (erf form) instead of the sigmoid
  int n_tiles;
  int use_raw;        // 1: runs of rows go through the raw ring; 0: all rows read from global
  int raw_stage;      // bytes of one raw stage
  int nraw;           // raw stages (4 .. kMaxRaw)
  int nstg;           // mode 0: staging buffers per epilogue group (1 or 2)
  int nacc;           // TMEM accumulators (2: the epilogue of a tile overlaps the next tile's MMAs)
  int acc_col;        // TMEM column of the first accumulator (the A operand takes columns 0 .. KP/2-1)
  int acc_stride;     // TMEM columns between the accumulators
  int box_n[3];       // mode 0: columns per TMA store box (32 -> 64B swizzle, 16 -> 32B swizzle)
  int off_raw, off_stage, off_misc;   // shared-memory layout (bytes)
  GemmJob jobs[3];
  int* err;
};

// K-major, 128-byte swizzle: element (row, k) of a [rows x KP] operand lives
// in K-atom k/64 at row*128 + ((k%64/8) ^ (row%8))*16 + (k%8)*2.
__device__ __forceinline__ uint32_t sw128_off(int row, int k, int rows) {
  return static_cast<uint32_t>((k >> 6) * rows * 128 + row * 128 + ((((k & 63) >> 3) ^ (row & 7)) << 4) + (k & 7) * 2);
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
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
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// named barriers: id 1 + g for epilogue group g (128 threads), id 3 for both groups
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
// the same with an AND of a predicate over the participating threads
__device__ __forceinline__ bool named_all(int id, int n, bool v) {
  uint32_t r;
  asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
               : "=r"(r) : "r"(v ? 1u : 0u), "r"(id), "r"(n) : "memory");
  return r != 0;
}
__device__ __forceinline__ bool warp_all_ok(bool v) { return __all_sync(0xffffffffu, v); }

__device__ __forceinline__ float sigmoid_fast(float v) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * v));
  return fmaf(0.5f, t, 0.5f);
}

__global__ void __launch_bounds__(kThreads, 1)
rib_token_gemm_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                      const __grid_constant__ CUtensorMap tm2, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int KP = p.KP, K = p.K;
  // this CTA's job, selected without dynamic indexing (which would put the
  // whole struct in local memory)
  const GemmJob job = blockIdx.y == 0 ? p.jobs[0] : (blockIdx.y == 1 ? p.jobs[1] : p.jobs[2]);
  const int N = job.N;
  const int box_n = blockIdx.y == 0 ? p.box_n[0] : (blockIdx.y == 1 ? p.box_n[1] : p.box_n[2]);
  const CUtensorMap* tmap = blockIdx.y == 0 ? &tm0 : (blockIdx.y == 1 ? &tm1 : &tm2);
  const int rowbytes = K * 2;

  uint8_t* sW = smem;
  uint8_t* sRaw = smem + p.off_raw;
  uint8_t* sStage = smem + p.off_stage;
  uint8_t* misc = smem + p.off_misc;
  // per raw stage: source row of each of its 32 rows (-1: zero row) and raw
  // offset (-1: not in the raw buffer)
  long long* s_src = reinterpret_cast<long long*>(misc);                  // [kMaxRaw][32]
  int* s_roff = reinterpret_cast<int*>(misc + kMaxRaw * kSR * 8);         // [kMaxRaw][32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc + kMaxRaw * kSR * 12);
  uint64_t* raw_full = bars;                 // [kMaxRaw]
  uint64_t* raw_free = bars + kMaxRaw;       // [kMaxRaw]
  uint64_t* a_full = bars + 2 * kMaxRaw;     // [2] per K half of the TMEM operand
  uint64_t* a_free = a_full + 2;             // [2]
  uint64_t* acc_full = a_full + 4;           // [2]
  uint64_t* acc_free = a_full + 6;           // [2]
  uint64_t* done = a_full + 8;
  uint64_t* w_ready = a_full + 9;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(a_full + 10);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(tmem_holder + 1);

  __shared__ float s_bias[256];
  __shared__ int s_runs[kMaxRaw][3 * kSR];   // per stage and run: first row, end row, raw offset of the first row
  __shared__ int s_nruns[kMaxRaw];
  __shared__ int s_fast[kMaxRaw];   // 1: the stage holds 32 consecutive rows of A at raw offset r * rowbytes
  for (int i = tid; i < 256; i += kThreads) s_bias[i] = (job.bias && i < p.n_valid) ? job.bias[i] : 0.f;
  if (tid == 0) {
    for (int i = 0; i < kMaxRaw; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_free[i], 1);   // the warp of the stage's lane quarter
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], 4);     // the four warps of a K half
      mbar_init(&a_free[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_free[i], kEpiThreads / 32);
    }
    mbar_init(done, 1);
    mbar_init(w_ready, kEpiThreads / 32);
    *abort_flag = 0u;
    tmem_holder[2] = 0u;   // abort word of the teardown drains (never raised)
    fence_barrier_init();
    if (p.mode == 0) tma_prefetch_desc(tmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  // zero W' (its K padding and zero columns stay zero)
  for (int i = tid; i < p.off_raw / 16; i += kThreads) reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtx wc{abort_flag, p.err};
  const WaitCtx drain{reinterpret_cast<volatile uint32_t*>(tmem_holder + 2), p.err};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int it = 0, issued = 0;   // issued: raw stages whose copies were started
    bool stop = false;
    for (int tile = blockIdx.x; tile < p.n_tiles && !stop; tile += gridDim.x, ++it) {
      const long long t0 = static_cast<long long>(tile) * kTile;
      int b0 = 0, y0 = 0, x0 = 0;
      if (p.mode == 0) {
        const long long hw = static_cast<long long>(p.Hp) * p.Wp;
        b0 = static_cast<int>(t0 / hw);
        const long long rem = t0 - static_cast<long long>(b0) * hw;
        y0 = static_cast<int>(rem / p.Wp);
        x0 = static_cast<int>(rem - static_cast<long long>(y0) * p.Wp);
      }
      // fast path: the tile is one run of 128 consecutive rows of A whose
      // quarter tiles meet the bulk copy's 16-byte rules (every tile with no
      // padded token on a map with C % 8 == 0 or an even first row, every full
      // pointwise tile): lane 0 issues the four stage copies with no per-row
      // tables
      // (the source rows of valid tokens increase by one from token to token,
      // across padded columns too, so a tile whose first and last tokens are
      // valid and 127 source rows apart has no padded token and one run)
      long long s0t = -1;
      if (p.use_raw) {
        auto src_of = [&](long long t) -> long long {
          if (t >= p.T) return -1;
          if (p.mode != 0) return t;
          const long long hw = static_cast<long long>(p.Hp) * p.Wp;
          const int b = static_cast<int>(t / hw);
          const long long rem = t - static_cast<long long>(b) * hw;
          const int y = static_cast<int>(rem / p.Wp);
          const int x = static_cast<int>(rem - static_cast<long long>(y) * p.Wp);
          return (y < p.H && x < p.W) ? (static_cast<long long>(b) * p.H + y) * p.W + x : -1;
        };
        const long long sa = src_of(t0), se = src_of(t0 + kTile - 1);
        if (sa >= 0 && se >= 0 && se - sa == kTile - 1) s0t = sa;
        if (s0t >= 0 && ((s0t * rowbytes) % 16 != 0 || (kSR * rowbytes) % 16 != 0)) s0t = -1;
      }
      if (s0t >= 0) {
        if (lane == 0) {
          for (int qq = 0; qq < kTile / kSR; ++qq) {
            const int ss = (kTile / kSR) * it + qq, st = ss % p.nraw, use = ss / p.nraw;
            if (use > 0 && !mbar_wait(&raw_free[st], (use - 1) & 1, wc, SITE_G_RAW_FREE)) {
              stop = true;
              break;
            }
            s_fast[st] = 1;
            const uint32_t bytes = static_cast<uint32_t>(kSR * rowbytes);
            mbar_arrive_expect_tx(&raw_full[st], bytes);
            bulk_load(sRaw + st * p.raw_stage, p.A + (s0t + kSR * qq) * K, bytes, &raw_full[st]);
            issued = ss + 1;
          }
        }
        stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
        issued = __shfl_sync(0xffffffffu, issued, 0);
        continue;
      }
      for (int qq = 0; qq < kTile / kSR; ++qq) {
        const int ss = (kTile / kSR) * it + qq;   // raw stage sequence number
        const int st = ss % p.nraw, use = ss / p.nraw;
        if (use > 0 && !warp_all_ok(mbar_wait(&raw_free[st], (use - 1) & 1, wc, SITE_G_RAW_FREE))) {
          stop = true;
          break;
        }
        long long* src_t = s_src + st * kSR;
        int* roff_t = s_roff + st * kSR;
        int* runs = s_runs[st];
        // source row of each row of the quarter tile: the padded-image token
        // maps to the unpadded map (-1 in the padding and past the last row)
        const int rt = kSR * qq + lane;
        long long src = -1;
        if (t0 + rt < p.T) {
          if (p.mode == 0) {
            int x = x0 + rt, y = y0, b = b0;
            if (x >= p.Wp) {
              y += x / p.Wp;
              x -= (x / p.Wp) * p.Wp;
              if (y >= p.Hp) {
                b += y / p.Hp;
                y -= (y / p.Hp) * p.Hp;
              }
            }
            if (y < p.H && x < p.W) src = (static_cast<long long>(b) * p.H + y) * p.W + x;
          } else {
            src = t0 + rt;
          }
        }
        src_t[lane] = src;
        // common case: the whole quarter tile is one run of consecutive rows of A
        const long long s0 = __shfl_sync(0xffffffffu, src, 0);
        const bool one_run = p.use_raw && __all_sync(0xffffffffu, s0 >= 0 && src == s0 + lane);
        if (one_run) {
          // bulk part [rb, re): 16-byte aligned source start and byte count
          const int rb = (s0 * rowbytes) % 16 != 0 ? 1 : 0;
          const int re = ((kSR - rb) * rowbytes) % 16 != 0 ? kSR - 1 : kSR;
          const int dst = (rb * rowbytes + 15) & ~15;
          roff_t[lane] = (lane >= rb && lane < re) ? dst + (lane - rb) * rowbytes : -1;
          __syncwarp();
          if (lane == 0) {
            s_fast[st] = 0;
            const uint32_t bytes = static_cast<uint32_t>((re - rb) * rowbytes);
            mbar_arrive_expect_tx(&raw_full[st], bytes);
            bulk_load(sRaw + st * p.raw_stage + dst, p.A + (s0 + rb) * K, bytes, &raw_full[st]);
          }
        } else {
          roff_t[lane] = -1;
          // rows that continue the run of the row above (source row + 1)
          const long long prev = __shfl_up_sync(0xffffffffu, src, 1);
          const unsigned cont = __ballot_sync(0xffffffffu, lane > 0 && src >= 0 && prev >= 0 && src == prev + 1);
          const unsigned startm = __ballot_sync(0xffffffffu, src >= 0) & ~cont;
          __syncwarp();
          if (p.use_raw && lane == 0) {
            // runs of rows contiguous in A: a valid row that does not continue
            // starts one, which ends at the next row that does not continue.
            // Bulk-copy the part of a run that meets the 16-byte rules; rows
            // outside it stay at -1 and are read from global memory.
            int n_runs = 0;
            for (unsigned msk = startm; msk; msk &= msk - 1) {
              const int r0 = __ffs(msk) - 1;
              const long long sr0 = src_t[r0];
              int e = kSR;
              if (r0 + 1 < kSR) {
                const unsigned rest = ~cont >> (r0 + 1);
                if (rest != 0u) e = r0 + __ffs(rest);
              }
              int rb = r0, re = e;
              if ((sr0 * rowbytes) % 16 != 0) ++rb;
              if (re > rb && ((re - rb) * rowbytes) % 16 != 0) --re;
              if (re > rb) {
                runs[3 * n_runs] = rb;
                runs[3 * n_runs + 1] = re;
                runs[3 * n_runs + 2] = (rb * rowbytes + 16 * n_runs + 15) & ~15;   // raw offset of row rb
                ++n_runs;
              }
            }
            s_nruns[st] = n_runs;
          }
          __syncwarp();
          const int n_runs = p.use_raw ? s_nruns[st] : 0;
          // raw offset of each row inside a run's bulk part
          for (int k = 0; k < n_runs; ++k)
            if (lane >= runs[3 * k] && lane < runs[3 * k + 1]) roff_t[lane] = runs[3 * k + 2] + (lane - runs[3 * k]) * rowbytes;
          __syncwarp();
          if (lane == 0) {
            s_fast[st] = 0;
            uint32_t tx = 0;
            for (int k = 0; k < n_runs; ++k) tx += static_cast<uint32_t>((runs[3 * k + 1] - runs[3 * k]) * rowbytes);
            mbar_arrive_expect_tx(&raw_full[st], tx);
            uint8_t* dst = sRaw + st * p.raw_stage;
            for (int k = 0; k < n_runs; ++k) {
              const int rb = runs[3 * k], re = runs[3 * k + 1];
              bulk_load(dst + runs[3 * k + 2], p.A + src_t[rb] * K, static_cast<uint32_t>((re - rb) * rowbytes),
                        &raw_full[st]);
            }
          }
        }
        __syncwarp();
        issued = ss + 1;
      }
    }
    // drain: the copies of the last raw stages have landed before the CTA may exit
    if (lane == 0) {
      for (int ss = issued - p.nraw > 0 ? issued - p.nraw : 0; ss < issued; ++ss)
        mbar_wait(&raw_full[ss % p.nraw], (ss / p.nraw) & 1, drain, SITE_G_DRAIN);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = p.a_f16 ? idesc_f16(128, N, false, false) : idesc_bf16(128, N, false, false);
      const uint32_t w0 = smem_u32(sW);
      const int ks_half = KP / 32;   // K steps per half of the operand
      int it = 0;
      // W' staged by the epilogue warps
      bool ok = mbar_wait(w_ready, 0, wc, SITE_G_W_READY);
      for (int tile = blockIdx.x; ok && tile < p.n_tiles; tile += gridDim.x, ++it) {
        const int ab = p.nacc == 2 ? (it & 1) : 0;       // accumulator
        const int ua = p.nacc == 2 ? (it >> 1) : it;     // earlier tiles through it
        if (ua > 0 && !(ok = mbar_wait(&acc_free[ab], (ua - 1) & 1, wc, SITE_G_ACC_FREE))) break;
        const uint32_t acc = tmem + static_cast<uint32_t>(p.acc_col + ab * p.acc_stride);
        for (int h = 0; h < 2; ++h) {
          // K half h of the tile's operand written to TMEM by the reformat warps
          if (!(ok = mbar_wait(&a_full[h], it & 1, wc, SITE_G_A_FULL))) break;
          tc_fence_after();
          for (int ks = h * ks_half; ks < (h + 1) * ks_half; ++ks) {
            // K step ks: A columns 8 ks .. 8 ks + 7 (bf16 pairs); W' atom ks/4, 32-byte offset (ks%4)
            const uint32_t kw = (ks >> 2) * (N * 128) + (ks & 3) * 32;
            umma_ts(acc, tmem + 8u * ks, make_sdesc(w0 + kw, 16, 1024, SW_128B), idesc, ks > 0 ? 1u : 0u);
          }
          umma_commit(&a_free[h]);
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
      }
      umma_commit(done);
      mbar_wait(done, 0, drain, SITE_G_DRAIN);
    }
  } else if (warp < kEpi0) {
    // ------------------------------------------------------------ reformat
    // Warp w serves TMEM lane quarter w % 4, i.e. tile rows 32 (w % 4) ..
    // 32 (w % 4) + 31, which are raw stage w % 4 of each tile, and writes the
    // operand's two K halves in turn, each once the MMAs of the previous tile
    // have read it. Thread = tile row = TMEM lane: it reads its row's bf16
    // pairs from the raw stage (8-byte loads; rows 2K bytes apart,
    // conflict-free for 16 lanes at a time) and stores them to TMEM as the A
    // operand (column = K pair), zeros past K.
    const int quarter = warp & 3;
    const int hwords = KP / 4;               // 32-bit columns per K half
    const int kw = K / 2;                    // columns with data (K is even)
    const uint32_t ta = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++it) {
      const int ss = (kTile / kSR) * it + quarter, st = ss % p.nraw;
      if (!(ok = warp_all_ok(mbar_wait(&raw_full[st], (ss / p.nraw) & 1, wc, SITE_G_RAW_FULL)))) break;
      const bool fast = s_fast[st] != 0;
      int roff;
      long long src;
      if (fast) {
        roff = lane * rowbytes;   // 32 consecutive rows at raw offset r * rowbytes
        src = 0;
      } else {
        roff = s_roff[st * kSR + lane];
        src = s_src[st * kSR + lane];
      }
      const uint8_t* raw = sRaw + st * p.raw_stage + (roff > 0 ? roff : 0);
      const uint2* grow = reinterpret_cast<const uint2*>(p.A + (src > 0 ? src : 0) * K);
      for (int half = 0; half < 2 && ok; ++half) {
        const int c0 = half * hwords;          // first column of this half
        const int nv = kw - c0;                // columns of this half with data (even; may exceed hwords)
        // the MMAs of the previous tile have read this half
        if (it > 0 && !(ok = warp_all_ok(mbar_wait(&a_free[half], (it - 1) & 1, wc, SITE_G_A_FREE)))) break;
        tc_fence_after();
        for (int c = 0; c < hwords; c += 16) {
          uint32_t v[16];
          if (fast && c + 16 <= nv) {
            // whole chunk inside the row: eight independent loads, no branches
            // (the nested branches below serialise them: 3x slower)
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const uint2 x = *reinterpret_cast<const uint2*>(raw + (c0 + c + j) * 4);
              v[j] = x.x;
              v[j + 1] = x.y;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const int wd = c0 + c + j;   // even; kw even, so wd + 1 < kw too
              uint2 x = make_uint2(0u, 0u);
              if (wd < kw) {
                if (roff >= 0) x = *reinterpret_cast<const uint2*>(raw + wd * 4);
                else if (src >= 0) x = __ldg(grow + wd / 2);
              }
              v[j] = x.x;
              v[j + 1] = x.y;
            }
          }
          tmem_st16(ta + static_cast<uint32_t>(c0 + c), v);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[half]);
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&raw_free[st]);   // the stage's rows have been read
    }
  } else {
    // ------------------------------------------------------------ W' staging
    // (while the producer and the reformat warps bring in the first tiles):
    // item i = (k chunk, column c) gathers eight k of weight column c into
    // one 16-byte chunk of row n of the K-major operand (n = c for the gate,
    // the head-padded column for the projections); consecutive threads take
    // consecutive columns (coalesced loads), items are independent
    {
      const int et = tid - kEpi0 * 32;
      const uint16_t* Wt = static_cast<const uint16_t*>(job.Wt);
      const int items = ((K + 7) / 8) * p.w_cols;
#pragma unroll 4
      for (int i = et; i < items; i += kEpiThreads) {
        const int kc = i / p.w_cols;
        const int c = i - kc * p.w_cols;
        const int k0 = 8 * kc;
        const int n = p.mode == 0 ? (c / p.dh) * job.DP + (c % p.dh) : c;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t lo = (k0 + 2 * e < K) ? __ldg(Wt + static_cast<size_t>(k0 + 2 * e) * p.w_cols + c) : 0u;
          const uint32_t hi = (k0 + 2 * e + 1 < K) ? __ldg(Wt + static_cast<size_t>(k0 + 2 * e + 1) * p.w_cols + c) : 0u;
          // bf16 weights; as fp16 for an fp16 map (exact in fp16's normal range, saturating)
          w[e] = p.a_f16 ? pack_f16x2_sat(__uint_as_float(lo << 16), __uint_as_float(hi << 16)) : (lo | (hi << 16));
        }
        if (n < N) *reinterpret_cast<uint4*>(sW + sw128_off(n, k0, N)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(w_ready);
    }
    // ------------------------------------------------------------ epilogue
    const int g = (warp - kEpi0) >> 2;            // group: boxes g, g + kEpiGroups, ...
    const int quarter = warp & 3;                 // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;          // token row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const bool leader = (warp - kEpi0) % 4 == 0 && lane == 0;   // issues the group's stores
    const int bar_g = 1 + g;
    const int box_bytes = kTile * box_n * 2;
    uint8_t* stage_g = sStage + g * p.nstg * box_bytes;    // mode 0: nstg buffers per group
    int it = 0, box_ctr = 0;
    for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++it) {
      const int ab = p.nacc == 2 ? (it & 1) : 0;
      const int ua = p.nacc == 2 ? (it >> 1) : it;
      // one outcome for all the epilogue warps (they share named barriers)
      const bool ok = named_all(1 + kEpiGroups, kEpiThreads, mbar_wait(&acc_full[ab], ua & 1, wc, SITE_G_ACC_FULL));
      tc_fence_after();
      const long long t0 = static_cast<long long>(tile) * kTile;
      const long long rows = (p.T - t0) < kTile ? (p.T - t0) : kTile;
      if (!ok) break;
      const uint32_t acc = tmem + static_cast<uint32_t>(p.acc_col + ab * p.acc_stride) + lane_off;
      if (p.mode == 0) {
        const float s = job.scale;
        for (int c0 = g * box_n; c0 < N; c0 += kEpiGroups * box_n) {
          // box [c0, c0 + box_n): TMEM -> registers
          uint32_t v[32];
          if (box_n == 32) {
            tmem_ld32(acc + c0, v);
          } else {
            tmem_ld16(acc + c0, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
          }
          tmem_wait_ld();
          uint8_t* sb = stage_g + (p.nstg == 2 ? (box_ctr & 1) : 0) * box_bytes;
          // the store issued from this buffer nstg boxes ago has read it
          if (leader) {
            if (p.nstg == 2) bulk_wait_read1();
            else bulk_wait_read0();
          }
          named_sync(bar_g, 128);
#pragma unroll
          for (int q = 0; q < 4; ++q) {      // 16-byte groups of 8 columns
            if (8 * q < box_n) {
              const int c = c0 + 8 * q;
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                f[e] = __uint_as_float(v[8 * q + e]) * s;
                if (job.ones_col >= 0 && ((c + e) & (job.DP - 1)) >= job.ones_col) f[e] = 1.f;
              }
              uint4 o;
              if (job.out_f16) {
                o = make_uint4(pack_f16x2_sat(f[0], f[1]), pack_f16x2_sat(f[2], f[3]), pack_f16x2_sat(f[4], f[5]),
                               pack_f16x2_sat(f[6], f[7]));
              } else {
                o = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                               pack_bf16x2(f[6], f[7]));
              }
              // TMA swizzle of the box's rows: 16-byte chunk index XOR
              // ((row / 2) % 4) for 64-byte rows, XOR ((row / 4) % 2) for 32-byte rows
              uint32_t off;
              if (box_n == 32) off = row * 64 + ((q ^ ((row >> 1) & 3)) << 4);
              else off = row * 32 + ((q ^ ((row >> 2) & 1)) << 4);
              *reinterpret_cast<uint4*>(sb + off) = o;
            }
          }
          fence_proxy_async_smem();
          named_sync(bar_g, 128);
          if (leader) {
            tma_store_2d(tmap, sb, c0, static_cast<int>(t0));
            bulk_commit();
          }
          ++box_ctr;
        }
      } else {
        // the previous tile's bulk store has read the staging rows
        if (tid == kEpi0 * 32) bulk_wait_read0();
        named_sync(1 + kEpiGroups, kEpiThreads);
        for (int c0 = 32 * g; c0 < p.n_real; c0 += 32 * kEpiGroups) {
          uint32_t v[32];
          tmem_ld32(acc + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 8; ++q) {     // 8 groups of 4 columns
            const int c = c0 + 4 * q;
            if (c < p.n_real) {
              float gv[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float a = __uint_as_float(v[4 * q + e]) + s_bias[c + e];
                gv[e] = p.gelu ? 0.5f * a * (1.f + erff(a * 0.70710678118654752f)) : sigmoid_fast(a);
              }
              *reinterpret_cast<uint2*>(sStage + (row * p.n_real + c) * 2) =
                  job.out_f16 ? make_uint2(pack_f16x2_sat(gv[0], gv[1]), pack_f16x2_sat(gv[2], gv[3]))
                              : make_uint2(pack_bf16x2(gv[0], gv[1]), pack_bf16x2(gv[2], gv[3]));
            }
          }
        }
      }
      // accumulator drained: the MMA of tile it + 2 may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_free[ab]);
      if (p.mode != 0) {
        fence_proxy_async_smem();
        named_sync(1 + kEpiGroups, kEpiThreads);
        if ((rows * p.n_real * 2) % 16 == 0) {
          if (tid == kEpi0 * 32) {
            bulk_store(static_cast<__nv_bfloat16*>(job.out) + t0 * p.n_real, sStage,
                       static_cast<uint32_t>(rows * p.n_real * 2));
            bulk_commit();
          }
        } else if (g == 0 && row < rows) {
          // ragged last tile whose byte count is not a multiple of 16: plain stores
          const uint2* src = reinterpret_cast<const uint2*>(sStage + row * p.n_real * 2);
          uint2* dst = reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(job.out) + (t0 + row) * p.n_real);
          for (int q = 0; q < p.n_real / 4; ++q) dst[q] = src[q];
        }
      }
    }
    if (leader || tid == kEpi0 * 32) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_token_gemm(const GemmLaunch& g, cudaStream_t stream) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
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
  p.n_valid = g.n_valid > 0 ? g.n_valid : g.n_real;
  p.a_f16 = g.a_f16;
  p.gelu = g.gelu;
  p.w_cols = g.w_cols;
  p.n_tiles = static_cast<int>((p.T + kTile - 1) / kTile);
  int n_max = 16;
  for (int i = 0; i < 3; ++i) {
    p.jobs[i] = g.jobs[i];
    p.box_n[i] = (g.jobs[i].N % 32 == 0) ? 32 : 16;
    if (i < g.njobs) n_max = g.jobs[i].N > n_max ? g.jobs[i].N : n_max;
  }
  p.err = device_error_word();
  if (p.n_tiles == 0) return cudaSuccess;
  // TMEM: the A operand (KP/2 columns of bf16 pairs) | one or two accumulators
  auto up = [](int v, int a) { return (v + a - 1) / a * a; };
  p.acc_col = up(p.KP / 2, 32);
  p.acc_stride = up(n_max, 32);
  p.nacc = p.acc_col + 2 * p.acc_stride <= 512 ? 2 : 1;
  if (p.acc_col + p.acc_stride > 512) return cudaErrorInvalidConfiguration;
  // shared memory: W' | raw ring | staging | tables + barriers
  const int w_bytes = up(n_max * p.KP * 2, 1024);
  p.raw_stage = up(kSR * g.K * 2 + 16 * kSR + 16, 128);
  const int misc_bytes = kMaxRaw * kSR * 12 + 24 * 8;
  // bulk copies need a 16-byte aligned source
  p.use_raw = (reinterpret_cast<uintptr_t>(g.A) % 16) == 0 ? 1 : 0;
  auto stage_for = [&](int nstg) { return g.mode == 0 ? kEpiGroups * nstg * kTile * 32 * 2 : up(kTile * g.n_real * 2, 1024); };
  auto total_for = [&](int nraw, int nstg) {
    return w_bytes + up(p.use_raw ? nraw * p.raw_stage : 0, 1024) + stage_for(nstg) + misc_bytes + 1024;
  };
  // the deepest raw ring (4 .. 8 stages: at least one tile) with two staging
  // buffers per group, else with one
  p.nraw = 0;
  for (int nstg = 2; nstg >= 1 && p.nraw == 0; --nstg)
    for (int nraw = kMaxRaw; nraw >= 4; --nraw)
      if (total_for(nraw, nstg) <= kSmemLimit) {
        p.nraw = nraw;
        p.nstg = nstg;
        break;
      }
  if (p.nraw == 0 && p.use_raw) {
    p.use_raw = 0;   // large K: rows read straight from global memory
    p.nraw = 4;
    p.nstg = total_for(4, 2) <= kSmemLimit ? 2 : 1;
  }
  int total = total_for(p.nraw, p.nstg);
  if (total > kSmemLimit) return cudaErrorInvalidConfiguration;
  p.off_raw = w_bytes;
  p.off_stage = p.off_raw + up(p.use_raw ? p.nraw * p.raw_stage : 0, 1024);
  p.off_misc = p.off_stage + stage_for(p.nstg);
  // at least half the shared memory: one CTA per SM (each allocates all of TMEM)
  if (total < 116 * 1024) total = 116 * 1024;
  CUtensorMap maps[3];
  std::memset(maps, 0, sizeof(maps));
  if (g.mode == 0) {
    for (int j = 0; j < g.njobs; ++j) {
      const uint64_t dims[2] = {uint64_t(g.jobs[j].N), uint64_t(p.T)};
      const uint64_t strides[1] = {uint64_t(g.jobs[j].N) * 2};
      const uint32_t box[2] = {uint32_t(p.box_n[j]), uint32_t(kTile)};
      if (encode_tiled(&maps[j], g.jobs[j].out_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                       g.jobs[j].out, dims, strides, box,
                       p.box_n[j] == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(rib_token_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, total);
  if (e != cudaSuccess) return e;
  // one CTA per SM; the persistent grid is co-resident
  const int sms = sm_count();
  int gx = sms / g.njobs;
  if (gx < 1) gx = 1;
  if (gx > p.n_tiles) gx = p.n_tiles;
  dim3 grid(gx, g.njobs);
  rib_token_gemm_kernel<<<grid, kThreads, total, stream>>>(maps[0], maps[1], maps[2], p);
  return cudaGetLastError();
}

}  // namespace rib
