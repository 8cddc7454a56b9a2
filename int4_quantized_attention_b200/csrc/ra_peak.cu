// ra_peak.cu -- measurement hook: the dense INT8 tensor-core rate as the
// attention kernel can reach it.
//
// One CTA per SM; one thread issues back-to-back tcgen05.mma.kind::i8
// M128 x N x K32 instructions (N = 128, the attention kernel's shape, or
// 256) on fixed shared-memory operands in the same 128-byte-swizzled K-major
// layout the attention kernel uses, four K steps per accumulator as there,
// alternating between two TMEM accumulators.  The caller times the launch
// with CUDA events; the operation count is
// ctas * iters * 4 * 2 * 128 * N * 32.  The operands' values do not matter
// for the timing (the result is discarded).
#include <cuda_runtime.h>

#include "ra_internal.h"

namespace ra {
namespace {

constexpr int PEAK_THREADS = 128;
// A: 128 x 128 B (16 KB); B: up to 256 x 128 B (32 KB); barrier + TMEM slot
constexpr uint32_t PEAK_SMEM = 16384 + 32768 + 64;

__global__ void __launch_bounds__(PEAK_THREADS, 1) mma_i8_rate_kernel(int iters, int n, WsHeader* hdr,
                                                                       uint64_t limit) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 16384 + 32768);
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + 16384 + 32768 + 8);
  const int tid = threadIdx.x, warp = tid >> 5;
  // small codes, so every product is representable; any bytes would do
  for (int i = tid; i < (16384 + 32768) / 16; i += PEAK_THREADS)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0x01FF0201u + i, 0x02FE0103u, 0xFF01FE02u, 0x0301FF01u);
  fence_async_smem();
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *slot;
  if (tid == 0) {
    const uint32_t a = smem_u32(sm), b = smem_u32(sm + 16384);
    const uint32_t idesc = n == 256 ? make_idesc(2, 1, 1, 128, 256) : make_idesc(2, 1, 1, 128, 128);
    for (int it = 0; it < iters; ++it) {
      const uint32_t d = tbase + (it & 1) * 256;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) umma_i8(d, sw128_desc(a + 32 * kk), sw128_desc(b + 32 * kk), idesc, kk > 0);
    }
    umma_commit(bar);
    mbar_wait(bar, 0, limit, &hdr->err, 0x5101);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace

cudaError_t launch_mma_i8_rate(int n, int iters, int ctas, void* ws, cudaStream_t st) {
  // more than half the SM's shared memory: one CTA per SM, so the 512-column
  // TMEM allocation never waits for another CTA
  constexpr int smem_one_per_sm = 120 * 1024;
  static_assert(PEAK_SMEM + 1024 <= smem_one_per_sm, "operands fit");
  cudaError_t e = cudaFuncSetAttribute(mma_i8_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_one_per_sm);
  if (e != cudaSuccess) return e;
  mma_i8_rate_kernel<<<ctas, PEAK_THREADS, smem_one_per_sm, st>>>(iters, n, static_cast<WsHeader*>(ws),
                                                                  wait_limit());
  return cudaGetLastError();
}

}  // namespace ra

// ---------------------------------------------------------------- ex2 probe
// y[i] = the INT4 attention kernel's 2^x (ex2.approx.ftz.f32, ra::ex2) for
// x[i]: a test measures its relative error against float64, which bounds
// where the kernel's P code may differ from the exact decision.
namespace ra {
namespace {
__global__ void ex2_probe_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = ex2(x[i]);
}
}  // namespace

cudaError_t launch_ex2_probe(const float* x, float* y, int n, cudaStream_t st) {
  if (n > 0) ex2_probe_kernel<<<(n + 255) / 256, 256, 0, st>>>(x, y, n);
  return cudaGetLastError();
}
}  // namespace ra
