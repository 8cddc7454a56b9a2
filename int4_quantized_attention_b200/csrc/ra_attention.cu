// ra_attention.cu -- INT4 and FP16 attention forward on the sm_100a tensor
// cores (tcgen05.mma, accumulators in tensor memory).
//
// RotateAttention (arXiv 2607.02584) review page: quantised FlashAttention
// with online softmax (abstract); range-optimised P quantisation, P =
// exp(QK^T - max) in [0,1] mapped onto [-8, 7] with fixed scale 15 and
// zero-point -8 (Sec. 4.2 via the referee report, free-parameter ledger);
// FP16 attention as the mixed-precision fallback (abstract, Sec. 5.1).
//
// One CTA handles one (batch*head, 128-row query tile); its 4 warps own the
// 128 TMEM lanes (thread t = query row t).  Per 128-key tile j:
//   1. K tile and V^T tile are widened into 128-byte-swizzled K-major SMEM
//      operands (INT4 codes -> INT8, scaled by 16 so the nibble lands in the
//      high half of the byte; the factor 256 on S and 16 on P.V is exact and
//      folded into the dequantisation);
//   2. one thread issues S = Q K^T (kind::i8, int32 in TMEM columns 0..127);
//   3. each thread loads its S row, takes the running max in the log2
//      domain, and turns every logit into the unsigned P operand
//      w = rne(15 * 2^(x - m)) = code + 8 in [0, 15];
//   4. rows whose max moved rescale their int32 P.V accumulator in place
//      (only then: exp(m_old - m_new) = 1 exactly otherwise);
//   5. one thread issues O += W V (u8 x s8, int32 in TMEM columns 128..255).
// Feeding w = code + 8 as an unsigned operand makes the tensor core compute
// sum (code + 8) v = sum code*v + 8 * colsum(v): the zero-point correction is
// carried out inside the MMA, bit-identical to adding 8 x the V column sum.
// The normaliser is l = sum w (exact integers per tile), so the 1/15 cancels.
#include <cuda_fp16.h>
#include <cstdint>

#include "ra_internal.h"

namespace ra {
namespace {

constexpr uint32_t IDESC_QK = make_idesc(2, 1, 1, 128, 128);    // s32 += s8 x s8
constexpr uint32_t IDESC_PV = make_idesc(2, 0, 1, 128, 128);    // s32 += u8 x s8
constexpr uint32_t IDESC_F16 = make_idesc(1, 0, 0, 128, 128);   // f32 += f16 x f16
constexpr float LOG2E = 1.4426950408889634f;
constexpr float MAGIC = 12582912.0f;                            // 1.5 * 2^23
constexpr int MAGIC_BITS = 0x4B400000;

// Widen 8 packed INT4 codes (one 32-bit word, element 2b in the low nibble of
// byte b) into 8 int8 values 16*code, in element order.
__device__ __forceinline__ uint2 widen8(uint32_t w) {
  const uint32_t lo = (w << 4) & 0xF0F0F0F0u;   // 16*e0, 16*e2, 16*e4, 16*e6
  const uint32_t hi = w & 0xF0F0F0F0u;          // 16*e1, 16*e3, 16*e5, 16*e7
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

// One 64-byte packed row (128 codes) -> one 128-byte swizzled int8 row.
__device__ __forceinline__ void widen_row_sw128(uint8_t* tile, uint32_t row, const uint8_t* __restrict__ src) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int h = 0; h < 4; ++h) {          // 16 packed bytes = 32 codes = 2 chunks
    const uint4 u = __ldg(s + h);
    const uint2 a = widen8(u.x), b = widen8(u.y), c = widen8(u.z), d = widen8(u.w);
    *reinterpret_cast<uint4*>(tile + sw128_off(row, 2 * h)) = make_uint4(a.x, a.y, b.x, b.y);
    *reinterpret_cast<uint4*>(tile + sw128_off(row, 2 * h + 1)) = make_uint4(c.x, c.y, d.x, d.y);
  }
}

struct AttnSmem {
  static constexpr uint32_t Q = 0, K = 16384, V = 32768, P = 49152, BAR = 65536, SV = BAR + 64,
                            BYTES = SV + 512;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ---------------------------------------------------------------------------
// INT4 attention.
__global__ void __launch_bounds__(128, 1)
    int4_attn_kernel(Prob Pb, const uint8_t* __restrict__ q4, const uint8_t* __restrict__ k4,
                     const uint8_t* __restrict__ v4t, const float* __restrict__ sq, const float* __restrict__ sk,
                     const float* __restrict__ sv, __half* __restrict__ o, WsHeader* __restrict__ hdr,
                     uint32_t limit, int dbg_bh, int dbg_qt, int dbg_kv, int32_t* __restrict__ dbg_s,
                     int8_t* __restrict__ dbg_p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* Qs = sm + AttnSmem::Q;
  uint8_t* Ks = sm + AttnSmem::K;
  uint8_t* Vs = sm + AttnSmem::V;
  uint8_t* Ps = sm + AttnSmem::P;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + AttnSmem::BAR);   // 0: S done, 1: PV done, 2: drain
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + AttnSmem::BAR + 32);
  int* abort_flag = reinterpret_cast<int*>(sm + AttnSmem::BAR + 40);
  float* svs = reinterpret_cast<float*>(sm + AttnSmem::SV);

  const int tid = threadIdx.x, warp = tid >> 5;
  // the debug launch runs the single CTA (dbg_qt, dbg_bh) and stores no output
  const bool dbg_run = dbg_s != nullptr;
  const int qt = blockIdx.x + (dbg_run ? dbg_qt : 0), bh = blockIdx.y + (dbg_run ? dbg_bh : 0);
  const int N = Pb.N, N_pad = Pb.N_pad, nblk = N_pad / QK_BLOCK;
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
  svs[tid] = sv[(size_t)bh * D + tid];
  // Q tile: row tid of this query tile, widened into the swizzled operand.
  const int row = qt * TILE + tid;
  widen_row_sw128(Qs, tid, q4 + ((size_t)bh * N_pad + row) * (D / 2));
  const float sQ = sq[(size_t)bh * nblk + row / QK_BLOCK];
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const uint32_t tS = tbase, tO = tbase + 128;
  const uint32_t lane = (uint32_t)(warp * 32) << 16;
  const uint32_t qs_addr = smem_u32(Qs), ks_addr = smem_u32(Ks), vs_addr = smem_u32(Vs), ps_addr = smem_u32(Ps);

  float m = -INFINITY;   // running max, log2 domain
  float l = 0.0f;        // running sum of P codes + 8, rescaled
  const int ntiles = N_pad / TILE;
  const float* skb = sk + (size_t)bh * nblk;
  const bool dbg_cta = dbg_run && bh == dbg_bh && qt == dbg_qt;

  for (int j = 0; j < ntiles; ++j) {
    // --- 1. operands: K rows and V^T rows of this tile
    widen_row_sw128(Ks, tid, k4 + ((size_t)bh * N_pad + (size_t)j * TILE + tid) * (D / 2));
    widen_row_sw128(Vs, tid, v4t + ((size_t)bh * D + tid) * (N_pad / 2) + (size_t)j * (TILE / 2));
    fence_async_smem();
    __syncthreads();
    // --- 2. S = Q K^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_i8(tS, sw128_desc(qs_addr + 32 * kk), sw128_desc(ks_addr + 32 * kk), IDESC_QK, kk > 0);
      umma_commit(&bar[0]);
    }
    if (!mbar_wait(&bar[0], j & 1, limit, err, 0x1001)) *abort_flag = 1;
    if (__syncthreads_or(*abort_flag)) break;
    tc_fence_after();
    // --- 3. softmax on this thread's row
    uint32_t s[128];
#pragma unroll
    for (int c = 0; c < 8; ++c) tmem_ld16(tS + lane + 16 * c, *reinterpret_cast<uint32_t(*)[16]>(&s[16 * c]));
    tmem_wait_ld();
    const int nvalid = min(TILE, N - j * TILE);
    const float c0 = __fmul_rn(__fmul_rn(sQ, skb[2 * j]), LOG2E / (11.313708498984761f * 256.0f));
    const float c1 = __fmul_rn(__fmul_rn(sQ, skb[2 * j + 1]), LOG2E / (11.313708498984761f * 256.0f));
    int mx0 = INT_MIN, mx1 = INT_MIN;
#pragma unroll
    for (int n = 0; n < 64; ++n)
      if (n < nvalid) mx0 = max(mx0, (int)s[n]);
#pragma unroll
    for (int n = 64; n < 128; ++n)
      if (n < nvalid) mx1 = max(mx1, (int)s[n]);
    float tmax = __fmul_rn((float)mx0, c0);
    if (nvalid > 64) tmax = fmaxf(tmax, __fmul_rn((float)mx1, c1));
    const float m_new = fmaxf(m, tmax);
    const bool moved = (j > 0) && (m_new > m);
    const float alpha = moved ? ex2(m - m_new) : 1.0f;
    // --- 4. lazy rescale of the int32 P.V accumulator for rows whose max moved
    if (__any_sync(0xffffffffu, moved)) {
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t acc[16];
        tmem_ld16(tO + lane + 16 * c, acc);
        tmem_wait_ld();
        if (moved) {
#pragma unroll
          for (int e = 0; e < 16; ++e) acc[e] = (uint32_t)__float2int_rn(__int2float_rn((int)acc[e]) * alpha);
        }
        tmem_st16(tO + lane + 16 * c, acc);
      }
      tmem_wait_st();
    }
    m = m_new;
    // P operand w = rne(15 * 2^(S*c - m)) in [0, 15]; 0 for keys past N.
    const float negm = -m;
    unsigned L = 0;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      uint32_t wv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t bytes[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int n = 16 * ch + 4 * q + e;
          const float sf = __int_as_float((int)s[n] + MAGIC_BITS) - MAGIC;   // exact int -> float
          const float p = ex2(fmaf(sf, n < 64 ? c0 : c1, negm));
          const int w = __float_as_int(fmaf(15.0f, p, MAGIC)) - MAGIC_BITS;
          bytes[e] = n < nvalid ? (uint32_t)w : 0u;
        }
        wv[q] = bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24);
        L = __dp4a(wv[q], 0x01010101u, (unsigned)L);
      }
      *reinterpret_cast<uint4*>(Ps + sw128_off(tid, ch)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      if (dbg_cta && j == dbg_kv) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int n = 16 * ch + 4 * q + e;
            dbg_s[tid * TILE + n] = n < nvalid ? ((int)s[n] >> 8) : 0;
            dbg_p[tid * TILE + n] = n < nvalid ? (int8_t)((int)((wv[q] >> (8 * e)) & 0xFF) - 8) : (int8_t)-128;
          }
      }
    }
    l = fmaf(l, alpha, (float)L);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // --- 5. O += W V
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_i8(tO, sw128_desc(ps_addr + 32 * kk), sw128_desc(vs_addr + 32 * kk), IDESC_PV, (j > 0) || (kk > 0));
      umma_commit(&bar[1]);
    }
    if (!mbar_wait(&bar[1], j & 1, limit, err, 0x1002)) *abort_flag = 1;
    if (__syncthreads_or(*abort_flag)) break;
    tc_fence_after();
  }

  if (!*abort_flag) {
    // --- epilogue: O = acc * s_V / (16 l), fp16.  The TMEM loads are
    // warp-collective, so every lane loads; only rows < N store.
    const float inv = 1.0f / (16.0f * l);
    __half* orow = dbg_run ? nullptr : o + ((size_t)bh * N + (row < N ? row : 0)) * D;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t acc[16];
      tmem_ld16(tO + lane + 16 * c, acc);
      tmem_wait_ld();
      uint32_t hv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float a = (float)(int)acc[2 * e] * svs[16 * c + 2 * e] * inv;
        const float b = (float)(int)acc[2 * e + 1] * svs[16 * c + 2 * e + 1] * inv;
        const __half2 h2 = __floats2half2_rn(a, b);
        hv[e] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      if (row < N && !dbg_run) {
        uint4* dst = reinterpret_cast<uint4*>(orow + 16 * c);
        dst[0] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        dst[1] = make_uint4(hv[4], hv[5], hv[6], hv[7]);
      }
    }
  } else if (tid == 0) {
    // drain: wait (bounded) for every tensor-core operation issued so far
    umma_commit(&bar[2]);
    mbar_wait(&bar[2], 0, limit, err, 0x1003);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
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
                     uint32_t limit) {
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
__global__ void timeout_probe_kernel(WsHeader* hdr, uint32_t limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, limit, &hdr->err, 0x3001);
  }
}

}  // namespace

cudaError_t launch_int4_attention(const Prob& p, const uint8_t* q4, const uint8_t* k4, const uint8_t* v4t,
                                  const float* sq, const float* sk, const float* sv, __half* o, void* ws, int dbg_bh,
                                  int dbg_qtile, int dbg_kv, int32_t* dbg_s, int8_t* dbg_p, cudaStream_t st) {
  // 100 KB of dynamic shared memory keeps residency at <= 2 CTAs per SM, so
  // two 256-column TMEM allocations always fit in the SM's 512 columns.
  const int smem = 100 * 1024;
  cudaError_t e = cudaFuncSetAttribute(int4_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid = dbg_s ? dim3(1, 1) : dim3(p.N_pad / TILE, p.BH);
  int4_attn_kernel<<<grid, 128, smem, st>>>(
      p, q4, k4, v4t, sq, sk, sv, o, static_cast<WsHeader*>(ws), wait_limit(), dbg_bh, dbg_qtile, dbg_kv, dbg_s,
      dbg_p);
  return cudaGetLastError();
}

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
