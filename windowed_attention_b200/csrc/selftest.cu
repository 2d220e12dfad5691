// Diagnostics.
//
// 1. Make one bounded barrier wait run out on purpose. Every wait of the
// library's kernels is an mbarrier wait bounded in time: when it runs out,
// the kernel records the wait's site in the device error word, raises its
// CTA's abort flag and returns, and rib_device_error() reports
// RIB_ERR_TIMEOUT. This kernel exercises exactly that path with a short
// limit: one warp waits on a barrier that nothing ever arrives on, so the GPU
// never faults or hangs and the context stays usable afterwards.
//
// 2. The issue rate of tcgen05.mma. The attention kernels' products are
// narrow (N = 16 to 64, the head and rank widths), so how many instructions
// an SM retires per cycle, rather than their FLOPs, sets their floor. This
// kernel measures it: CTAs per SM and issuing threads per CTA as asked, each
// thread issuing a chain of M = 128, K = 16 products of width N (operands in
// shared memory, zero-filled; its own TMEM accumulator), timed with clock64
// from the first issue to the completion of the last.
#include <cuda_runtime.h>

#include "rib_internal.h"
#include "sm100.cuh"

namespace rib {

namespace {

constexpr int kSelftestSite = 901;

__global__ void selftest_wait_kernel(unsigned long long limit_ns, int* err) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // nothing arrives: phase 0 never completes
    abort_flag = 0u;
    fence_barrier_init();
  }
  __syncthreads();
  const WaitCtx wc{&abort_flag, err};
  if (!mbar_try_wait(&bar, 0)) mbar_wait_slow(&bar, 0, wc, kSelftestSite, limit_ns);
  __syncthreads();
}

constexpr int kRateSite = 902;

// cycles[(cta * issuers + i) * 2 + {0, 1}] = clock64 cycles of issuer i from
// its first MMA to its last issue, and to the completion of its chain;
// spans[cta * 3 + {0, 1, 2}] (if given) = the CTA's SM and the globaltimer
// before its first and after its last chain, to check that the CTAs of an
// SM ran at the same time.
__global__ void selftest_mma_rate_kernel(int issuers, int n, int mmas, uint32_t tmem_cols,
                                         unsigned long long* cycles, unsigned long long* spans, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  // A: 128 rows x 16 bf16 (4 KB), B: n rows x 16 bf16 (n * 32 bytes), both
  // K-major without swizzle: [8-row group][2 K core matrices][8 rows x 16 B]
  uint8_t* a_tile = smem;
  uint8_t* b_tile = smem + 4096;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 4096 + 8192);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 4096 + 8192 + 64);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + 4096 + 8192 + 72);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < (4096 + 8192) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    for (int i = 0; i < issuers; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  fence_proxy_async_smem();   // the zero fill, for the tensor core's reads
  if (warp == 0) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();   // the other CTAs of the SM allocate too
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, err};
  if (spans && threadIdx.x == 0) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    spans[blockIdx.x * 3] = smid;
    spans[blockIdx.x * 3 + 1] = globaltimer();
  }
  if (warp < issuers && lane == 0) {
    const uint32_t idesc = idesc_bf16(128, n, false, false);
    const uint64_t adesc = make_sdesc(smem_u32(a_tile), 128, 256, SW_NONE);
    const uint64_t bdesc = make_sdesc(smem_u32(b_tile), 128, 256, SW_NONE);
    const uint32_t d = tmem + static_cast<uint32_t>(warp * n);   // columns [warp n, warp n + n)
    const long long t0 = clock64();
    for (int k = 0; k < mmas; ++k) umma_ss(d, adesc, bdesc, idesc, k > 0 ? 1u : 0u);
    const long long t1 = clock64();
    umma_commit(&bars[warp]);
    const bool ok = mbar_wait(&bars[warp], 0, wc, kRateSite);
    const long long t2 = clock64();
    const size_t o = (static_cast<size_t>(blockIdx.x) * issuers + warp) * 2;
    cycles[o] = static_cast<unsigned long long>(t1 - t0);
    cycles[o + 1] = ok ? static_cast<unsigned long long>(t2 - t0) : 0ull;
  }
  tc_fence_before();
  __syncthreads();
  if (spans && threadIdx.x == 0) spans[blockIdx.x * 3 + 2] = globaltimer();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

}  // namespace

}  // namespace rib

using namespace rib;

extern "C" rib_status rib_selftest_mma_rate(int ctas_per_sm, int issuers_per_cta, int n, int mmas,
                                            unsigned long long* cycles, unsigned long long* spans,
                                            cudaStream_t stream) {
  if (ctas_per_sm < 1 || ctas_per_sm > 4)
    return fail(RIB_ERR_INVALID_ARG, "rib_selftest_mma_rate: ctas_per_sm must be in 1..4");
  if (issuers_per_cta < 1 || issuers_per_cta > 4)
    return fail(RIB_ERR_INVALID_ARG, "rib_selftest_mma_rate: issuers_per_cta must be in 1..4");
  if (n < 16 || n > 256 || n % 16 != 0)
    return fail(RIB_ERR_INVALID_ARG, "rib_selftest_mma_rate: n must be a multiple of 16 in 16..256");
  if (mmas < 1 || mmas > 65536) return fail(RIB_ERR_INVALID_ARG, "rib_selftest_mma_rate: mmas must be in 1..65536");
  if (!cycles) return fail(RIB_ERR_INVALID_ARG, "rib_selftest_mma_rate: cycles is null");
  // TMEM columns per CTA (a power of two; ctas_per_sm of them fit in 512)
  const uint32_t cols = ctas_per_sm == 1 ? 512u : (ctas_per_sm == 2 ? 256u : 128u);
  if (static_cast<uint32_t>(issuers_per_cta * n) > cols)
    return fail(RIB_ERR_INVALID_ARG, "rib_selftest_mma_rate: issuers_per_cta * n exceeds the CTA's TMEM columns "
                                     "(512 / ctas_per_sm, rounded down to a power of two)");
  int* err = device_error_word();
  if (!err) return fail(RIB_ERR_CUDA, "rib_selftest_mma_rate: no device error word");
  // shared memory sized so that no more than ctas_per_sm CTAs share an SM
  // (the operands need 13 KB and 1 KB of alignment slack)
  const int smem = (220 * 1024) / ctas_per_sm;
  // (and the largest shared-memory carveout, so that ctas_per_sm of them can)
  cudaError_t e = cudaFuncSetAttribute(selftest_mma_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(selftest_mma_rate_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return cuda_fail(e, "rib_selftest_mma_rate: shared memory attributes");
  selftest_mma_rate_kernel<<<sm_count() * ctas_per_sm, 32 * issuers_per_cta, smem, stream>>>(issuers_per_cta, n, mmas,
                                                                                             cols, cycles, spans, err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "rib_selftest_mma_rate launch");
  return RIB_OK;
}

extern "C" rib_status rib_selftest_wait_timeout(int limit_us, cudaStream_t stream) {
  if (limit_us < 1 || limit_us > 1000000)
    return fail(RIB_ERR_INVALID_ARG, "rib_selftest_wait_timeout: limit_us must be in 1..1000000");
  int* err = device_error_word();
  if (!err) return fail(RIB_ERR_CUDA, "rib_selftest_wait_timeout: no device error word");
  selftest_wait_kernel<<<1, 32, 0, stream>>>(static_cast<unsigned long long>(limit_us) * 1000ull, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "rib_selftest_wait_timeout launch");
  return RIB_OK;
}
