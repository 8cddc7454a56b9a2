// ra_attention.cu -- FP16 attention forward (the mixed-precision fallback)
// on the sm_100a tensor cores, and the bounded-wait probe kernel.
//
// RotateAttention (arXiv 2607.02584) review page: accuracy-sensitive
// attention calls (first/last denoising steps and DiT blocks) stay in FP16
// (abstract, Sec. 5.1); this is that path: FlashAttention over the RoPE-encoded
// fp16 Q and K with fp32 accumulation in tensor memory.
//
// One CTA per (batch*head, 128-row query tile); thread t = query row t = TMEM
// lane t.  Per 128-key tile: operands copied into 128-byte-swizzled K-major
// SMEM (fp16 rows are 256 bytes: two swizzle atoms), S = Q K^T on
// tcgen05.mma.kind::f16 into TMEM, online softmax in registers, P in fp16 to
// SMEM, O += P V into TMEM; rows whose max moved rescale O in place.
#include <cuda_fp16.h>
#include <cstdint>

#include "ra_internal.h"

namespace ra {
namespace {

constexpr uint32_t IDESC_F16 = make_idesc(1, 0, 0, 128, 128);   // f32 += f16 x f16
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ---------------------------------------------------------------------------
// FP16 attention (inputs position-encoded and V transposed by the FP16
// prologue).  fp16 operands: a 128-element row is 256 bytes, i.e. two
// 128-byte swizzle atoms ("K blocks") of 64 elements, 16 KB apart.
struct F16Smem {
  static constexpr uint32_t Q = 0, K = 32768, V = 65536, P = 98304, BAR = 131072, BYTES = BAR + 64;
};

__device__ __forceinline__ uint32_t f16_off(uint32_t row, uint32_t col) {   // element offset (bytes)
  return (col >> 6) * 16384u + sw128_off(row, (col & 63) >> 3) + (col & 7) * 2;
}

// Copy one 256-byte fp16 row from global into the two-atom swizzled layout.
__device__ __forceinline__ void copy_row_f16(uint8_t* tile, uint32_t row, const __half* __restrict__ src) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4*>(tile + f16_off(row, 8 * c)) = __ldg(s + c);
}

__device__ __forceinline__ uint64_t f16_desc(uint32_t base, int kk) {   // K step kk of 16 elements
  return sw128_desc(base + (kk >> 2) * 16384u + (kk & 3) * 32u);
}

__global__ void __launch_bounds__(128, 1)
    fp16_attn_kernel(Prob Pb, const __half* __restrict__ qr, const __half* __restrict__ kr,
                     const __half* __restrict__ vt, __half* __restrict__ o, WsHeader* __restrict__ hdr,
                     uint64_t limit) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* Qs = sm + F16Smem::Q;
  uint8_t* Ks = sm + F16Smem::K;
  uint8_t* Vs = sm + F16Smem::V;
  uint8_t* Ps = sm + F16Smem::P;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + F16Smem::BAR);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + F16Smem::BAR + 32);
  int* abort_flag = reinterpret_cast<int*>(sm + F16Smem::BAR + 40);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int qt = blockIdx.x, bh = blockIdx.y;
  const int N = Pb.N, N_pad = Pb.N_pad;
  DeviceErr* err = &hdr->err;
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_init(&bar[2], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 256);
    tmem_relinquish();
  }
  const int row = qt * TILE + tid;
  copy_row_f16(Qs, tid, qr + ((size_t)bh * N_pad + row) * D);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const uint32_t tS = tbase, tO = tbase + 128;
  const uint32_t lane = (uint32_t)(warp * 32) << 16;
  const uint32_t qs_addr = smem_u32(Qs), ks_addr = smem_u32(Ks), vs_addr = smem_u32(Vs), ps_addr = smem_u32(Ps);
  const float cs = LOG2E / 11.313708498984761f;   // log2(e) / sqrt(128)
  float m = -INFINITY, l = 0.0f;
  const int ntiles = N_pad / TILE;
  for (int j = 0; j < ntiles; ++j) {
    copy_row_f16(Ks, tid, kr + ((size_t)bh * N_pad + (size_t)j * TILE + tid) * D);
    copy_row_f16(Vs, tid, vt + ((size_t)bh * D + tid) * N_pad + (size_t)j * TILE);
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) umma_f16(tS, f16_desc(qs_addr, kk), f16_desc(ks_addr, kk), IDESC_F16, kk > 0);
      umma_commit(&bar[0]);
    }
    if (!mbar_wait(&bar[0], j & 1, limit, err, 0x2001)) *abort_flag = 1;
    if (__syncthreads_or(*abort_flag)) break;
    tc_fence_after();
    uint32_t s[128];
#pragma unroll
    for (int c = 0; c < 8; ++c) tmem_ld16(tS + lane + 16 * c, *reinterpret_cast<uint32_t(*)[16]>(&s[16 * c]));
    tmem_wait_ld();
    const int nvalid = min(TILE, N - j * TILE);
    float tmax = -INFINITY;
#pragma unroll
    for (int n = 0; n < 128; ++n)
      if (n < nvalid) tmax = fmaxf(tmax, __uint_as_float(s[n]));
    tmax *= cs;
    const float m_new = fmaxf(m, tmax);
    const bool moved = (j > 0) && (m_new > m);
    const float alpha = moved ? ex2(m - m_new) : 1.0f;
    if (__any_sync(0xffffffffu, moved)) {
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t acc[16];
        tmem_ld16(tO + lane + 16 * c, acc);
        tmem_wait_ld();
        if (moved) {
#pragma unroll
          for (int e = 0; e < 16; ++e) acc[e] = __float_as_uint(__uint_as_float(acc[e]) * alpha);
        }
        tmem_st16(tO + lane + 16 * c, acc);
      }
      tmem_wait_st();
    }
    m = m_new;
    const float negm = -m;
    float Lsum = 0.0f;
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) {   // 8 keys per 16-byte chunk
      uint32_t hv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int n = 8 * ch + 2 * e;
        const float p0 = n < nvalid ? ex2(fmaf(__uint_as_float(s[n]), cs, negm)) : 0.0f;
        const float p1 = n + 1 < nvalid ? ex2(fmaf(__uint_as_float(s[n + 1]), cs, negm)) : 0.0f;
        Lsum += p0 + p1;
        const __half2 h2 = __floats2half2_rn(p0, p1);
        hv[e] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      *reinterpret_cast<uint4*>(Ps + f16_off(tid, 8 * ch)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    }
    l = fmaf(l, alpha, Lsum);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_f16(tO, f16_desc(ps_addr, kk), f16_desc(vs_addr, kk), IDESC_F16, (j > 0) || (kk > 0));
      umma_commit(&bar[1]);
    }
    if (!mbar_wait(&bar[1], j & 1, limit, err, 0x2002)) *abort_flag = 1;
    if (__syncthreads_or(*abort_flag)) break;
    tc_fence_after();
  }
  if (!*abort_flag) {
    const float inv = 1.0f / l;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t acc[16];
      tmem_ld16(tO + lane + 16 * c, acc);
      tmem_wait_ld();
      if (row < N) {
        uint32_t hv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const __half2 h2 = __floats2half2_rn(__uint_as_float(acc[2 * e]) * inv, __uint_as_float(acc[2 * e + 1]) * inv);
          hv[e] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        uint4* dst = reinterpret_cast<uint4*>(o + ((size_t)bh * N + row) * D + 16 * c);
        dst[0] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        dst[1] = make_uint4(hv[4], hv[5], hv[6], hv[7]);
      }
    }
  } else if (tid == 0) {
    umma_commit(&bar[2]);
    mbar_wait(&bar[2], 0, limit, err, 0x2003);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

// A barrier nothing arms: the bounded wait must run out, record
// DEVERR_TIMEOUT and return.
__global__ void timeout_probe_kernel(WsHeader* hdr, uint64_t limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, limit, &hdr->err, 0x3001);
  }
}

}  // namespace

cudaError_t launch_fp16_attention(const Prob& p, __half* o, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(p);
  char* base = static_cast<char*>(ws);
  const int smem = F16Smem::BYTES + 1024;
  cudaError_t e = cudaFuncSetAttribute(fp16_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  fp16_attn_kernel<<<dim3(p.N_pad / TILE, p.BH), 128, smem, st>>>(
      p, reinterpret_cast<const __half*>(base + L.qr), reinterpret_cast<const __half*>(base + L.kr),
      reinterpret_cast<const __half*>(base + L.vt), o, static_cast<WsHeader*>(ws), wait_limit());
  return cudaGetLastError();
}

cudaError_t launch_timeout_probe(void* ws, cudaStream_t st) {
  timeout_probe_kernel<<<1, 32, 0, st>>>(static_cast<WsHeader*>(ws), wait_limit());
  return cudaGetLastError();
}

}  // namespace ra
