// ra_attention.cu -- FP16 attention forward (the mixed-precision fallback)
// on the sm_100a tensor cores, and the bounded-wait probe kernel.
//
// RotateAttention (arXiv 2607.02584) review page: accuracy-sensitive
// attention calls (first/last denoising steps and DiT blocks) stay in FP16
// (abstract, Sec. 5.1); this is that path: FlashAttention over the RoPE-encoded
// fp16 Q and K, P in fp16, fp32 accumulation in tensor memory.
//
// One CTA = one (batch*head, pair of 128-row query tiles A and B); 384
// threads:
//   warps 0-3 / 4-7   softmax of tile A / B; thread t = query row t = TMEM lane t
//   warp 8            bulk copies: the two Q tiles once, then the K tiles
//   warp 11           bulk copies of the V^T tiles
//   warps 9, 10       MMA issuers, one thread per query tile (warp 9 owns TMEM)
// The FP16 prologue writes Q, K and V^T as operand images: per 128-row tile,
// two 16 KB 128-byte-swizzled K-major atoms (elements 0..63 and 64..127 of
// every row), so each tile is one 32 KB bulk copy.  K and V^T have separate
// 2-stage rings: a K stage is free once both tiles' S MMAs have read it, a V
// stage once both tiles' P.V MMAs have.
// TMEM: S_A | S_B | O_A | O_B, 128 fp32 columns each.  The softmax threads
// load S_X(j), then store P_X(j) as fp16 pairs into the upper 64 columns of
// S_X, from where the P.V MMAs read their A operand.  Tile X's thread issues,
// per KV tile j: O_X += P_X(j) V(j) (once P_X(j) is stored), then S_X(j+1)
// (which overwrites the P columns, so it follows the P.V in issue order).
// MMAs of one thread complete in issue order: S_X(j+1) landing means P.V(j)
// has too, so the softmax may rescale O_X (fp32) right then.
// A 64-key half whose largest exponent is below -26 holds only P values that
// round to zero in fp16; its exponentials are skipped when that is so for
// every row of a warp (the fp16 operand is the same).
#include <cuda_fp16.h>
#include <cstdint>

#include "ra_internal.h"

namespace ra {
namespace {

namespace f16 {
constexpr int NUM_THREADS = 384;
constexpr int STAGES = 2;
constexpr int LAUNCH_REGS = 168, SOFTMAX_REGS = 208, ISSUE_REGS = 88;
static_assert(256 * SOFTMAX_REGS + 128 * ISSUE_REGS <= NUM_THREADS * LAUNCH_REGS, "register split");
constexpr uint32_t IDESC = make_idesc(1, 0, 0, 128, 128);   // f32 += f16 x f16
constexpr float LOG2E = 1.4426950408889634f;
constexpr float SKIP_BELOW = -26.0f;                        // 2^-26 rounds to fp16 zero
struct Smem {
  static constexpr uint32_t QA = 0, QB = 32768;            // 32 KB Q tiles
  static constexpr uint32_t K = 65536;                       // 2 x 32 KB
  static constexpr uint32_t V = 131072;                      // 2 x 32 KB
  static constexpr uint32_t BAR = 196608;
  static constexpr uint32_t BYTES = BAR + 512;
};
enum : int {
  B_KFULL = 0, B_KEMPTY = 2, B_VFULL = 4, B_VEMPTY = 6, B_QFULL = 8, B_SFULL = 9, B_PFULL = 11, B_ODONE = 13,
  B_DRAIN = 15, NBAR = 17
};
// K step kk (16 elements) of a two-atom operand tile
__device__ __forceinline__ uint64_t desc(uint32_t base, int kk) {
  return sw128_desc(base + (kk >> 2) * 16384u + (kk & 3) * 32u);
}
}  // namespace f16

__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(f16::NUM_THREADS, 1)
    fp16_attn_kernel(Prob Pb, const uint8_t* __restrict__ qimg, const uint8_t* __restrict__ kimg,
                     const uint8_t* __restrict__ vimg, __half* __restrict__ o, WsHeader* __restrict__ hdr,
                     uint64_t limit) {
  using namespace f16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Smem::BAR);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Smem::BAR + 8 * NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Smem::BAR + 8 * NBAR + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nt = Pb.N_pad / TILE;
  const int qt0 = 2 * blockIdx.x, bh = blockIdx.y;
  const bool hasB = qt0 + 1 < nt;
  DeviceErr* err = &hdr->err;

  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&bar[B_KFULL + i], 1);
      mbar_init(&bar[B_KEMPTY + i], hasB ? 2 : 1);
      mbar_init(&bar[B_VFULL + i], 1);
      mbar_init(&bar[B_VEMPTY + i], hasB ? 2 : 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[B_SFULL + i], 1);
      mbar_init(&bar[B_PFULL + i], 4);
      mbar_init(&bar[B_ODONE + i], 1);
      mbar_init(&bar[B_DRAIN + i], 1);
    }
    mbar_init(&bar[B_QFULL], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  if (warp < 8) {
    regs_inc<SOFTMAX_REGS>();
  } else {
    regs_dec<ISSUE_REGS>();
  }

  if (warp < 8) {
    // ------------------------------------------------------------ softmax
    const int X = warp >> 2, wq = warp & 3;
    if (X == 0 || hasB) {
      auto wait_all = [&](int b, uint32_t parity, uint32_t site) {
        return __all_sync(0xffffffffu, mbar_wait_abortable(&bar[b], parity, abort_flag, limit, err, site));
      };
      const int row = qt0 * TILE + X * TILE + (tid & 127);
      const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
      const uint32_t tS = tbase + X * 128 + lane_off, tO = tbase + 256 + X * 128 + lane_off;
      const float cs = LOG2E / 11.313708498984761f;   // log2(e) / sqrt(128)
      const int tail = Pb.N - (nt - 1) * TILE;        // valid keys in the last tile, 1..128
      float m = -INFINITY, l = 0.0f;
      bool ok = true;
      for (int j = 0; j < nt; ++j) {
        // S_X(j) has landed -- and with it P.V(j-1)
        if (!(ok = wait_all(B_SFULL + X, j & 1, 0x2101))) break;
        tc_fence_after();
        uint32_t s[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, s + 32 * c);
        tmem_wait_ld();
        const int nvalid = (j == nt - 1) ? tail : TILE;
        if (nvalid < TILE) {
#pragma unroll
          for (int n = 0; n < 128; ++n)
            if (n >= nvalid) s[n] = 0xFF800000u;   // -inf: out of the max and the sum
        }
        float mh[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          mh[c] = fmax3(__uint_as_float(s[16 * c]), __uint_as_float(s[16 * c + 1]), __uint_as_float(s[16 * c + 2]));
#pragma unroll
          for (int n = 3; n < 15; n += 2)
            mh[c] = fmax3(mh[c], __uint_as_float(s[16 * c + n]), __uint_as_float(s[16 * c + n + 1]));
          mh[c] = fmaxf(mh[c], __uint_as_float(s[16 * c + 15]));
        }
        const float mx0 = fmaxf(fmax3(mh[0], mh[1], mh[2]), mh[3]) * cs;
        const float mx1 = fmaxf(fmax3(mh[4], mh[5], mh[6]), mh[7]) * cs;
        const float m_new = fmaxf(m, fmaxf(mx0, mx1));
        const bool moved = j > 0 && m_new > m;
        const float alpha = moved ? ex2(m - m_new) : 1.0f;
        m = m_new;
        const float negm = -m;
        // rows whose max moved: O *= alpha (P.V(j-1) has landed, P.V(j) not issued)
        if (__any_sync(0xffffffffu, moved)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t acc[32];
            tmem_ld32(tO + 32 * c, acc);
            tmem_wait_ld();
            if (moved) {
#pragma unroll
              for (int e = 0; e < 32; ++e) acc[e] = __float_as_uint(__uint_as_float(acc[e]) * alpha);
            }
            tmem_st32(tO + 32 * c, acc);
          }
        }
        const bool zero_half[2] = {__all_sync(0xffffffffu, mx0 - m < SKIP_BELOW) != 0,
                                   __all_sync(0xffffffffu, mx1 - m < SKIP_BELOW) != 0};
        float lsum0 = 0.0f, lsum1 = 0.0f;   // row sum over even / odd keys
        uint32_t ph[64];   // P as fp16 pairs: ph[c] = keys 2c (low), 2c + 1
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (zero_half[h]) {
#pragma unroll
            for (int c = 32 * h; c < 32 * h + 32; ++c) ph[c] = 0u;
            continue;
          }
#pragma unroll
          for (int c = 32 * h; c < 32 * h + 32; ++c) {   // pairs of keys on packed fp32 pairs
            float x0, x1;
            fma2(x0, x1, __uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1]), cs, cs, negm, negm);
            const float p0 = ex2(x0), p1 = ex2(x1);
            add2(lsum0, lsum1, lsum0, lsum1, p0, p1);
            const __half2 h2 = __floats2half2_rn(p0, p1);
            ph[c] = *reinterpret_cast<const uint32_t*>(&h2);
          }
        }
        l = fmaf(l, alpha, lsum0 + lsum1);
        tmem_st32(tS + 64, ph);
        tmem_st32(tS + 96, ph + 32);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_PFULL + X]);
      }
      if (ok) ok = wait_all(B_ODONE + X, 0, 0x2102);
      if (ok) {
        // epilogue: O / l -> fp16 for rows < N; loads are warp-collective
        tc_fence_after();
        const float inv = 1.0f / l;
        const bool store = row < Pb.N && in_bounds(bh < Pb.BH, err, 0x2211);
        __half* orow = o + ((size_t)bh * Pb.N + (store ? row : 0)) * D;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t acc[32];
          tmem_ld32(tO + 32 * c, acc);
          tmem_wait_ld();
          uint32_t hv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const __half2 h2 =
                __floats2half2_rn(__uint_as_float(acc[2 * e]) * inv, __uint_as_float(acc[2 * e + 1]) * inv);
            hv[e] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_uint4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
          }
        }
      }
    }
  } else if (warp == 8 || warp == 11) {
    // ------------------------------------------------------------ bulk copies (warp 8: Q, K; warp 11: V^T)
    if (lane == 0) {
      const bool isK = warp == 8;
      const uint8_t* src = (isK ? kimg : vimg) + (size_t)bh * nt * 32768;
      const int FULL = isK ? B_KFULL : B_VFULL, EMPTY = isK ? B_KEMPTY : B_VEMPTY;
      const uint32_t base = isK ? Smem::K : Smem::V;
      // the grid covers the problem exactly: every copy below reads tiles
      // bh * nt + t with t < nt of an image of BH * nt tiles
      const bool ok_idx = in_bounds(bh < Pb.BH && qt0 + (hasB ? 2 : 1) <= nt, err, 0x2210);
      if (!ok_idx) *abort_flag = 1;   // every wait gives up; nothing is copied
      if (isK && ok_idx) {
        const uint8_t* qsrc = qimg + ((size_t)bh * nt + qt0) * 32768;
        mbar_expect_tx(&bar[B_QFULL], hasB ? 65536u : 32768u);
        bulk_g2s(sm + Smem::QA, qsrc, 32768, &bar[B_QFULL]);
        if (hasB) bulk_g2s(sm + Smem::QB, qsrc + 32768, 32768, &bar[B_QFULL]);
      }
      int issued = 0;
      for (int j = 0; ok_idx && j < nt; ++j) {
        const int st = j % STAGES;
        if (j >= STAGES &&
            !mbar_wait_abortable(&bar[EMPTY + st], ((j / STAGES) - 1) & 1, abort_flag, limit, err, 0x2201))
          break;
        mbar_expect_tx(&bar[FULL + st], 32768u);
        bulk_g2s(sm + base + st * 32768, src + (size_t)j * 32768, 32768, &bar[FULL + st]);
        issued = j + 1;
      }
      if (*abort_flag) {   // let every copy still in flight land before the CTA exits
        if (isK && ok_idx) mbar_wait(&bar[B_QFULL], 0, limit, err, 0x2203);
        for (int j = issued > STAGES ? issued - STAGES : 0; j < issued; ++j)
          mbar_wait(&bar[FULL + j % STAGES], (j / STAGES) & 1, limit, err, 0x2204);
      }
    }
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------ MMA issuers
    const int X = warp - 9;
    if (lane == 0 && (X == 0 || hasB)) {
      const uint32_t qa = smem_u32(sm + (X ? Smem::QB : Smem::QA));
      const uint32_t kb = smem_u32(sm + Smem::K), vb = smem_u32(sm + Smem::V);
      const uint32_t tS = tbase + X * 128, tO = tbase + 256 + X * 128;
      auto wait = [&](int b, uint32_t parity, uint32_t site) {
        return mbar_wait_abortable(&bar[b], parity, abort_flag, limit, err, site);
      };
      auto issue_S = [&](int j) {   // S_X(j) = Q_X K(j)^T, then release the K stage
        const uint32_t kt = kb + (j % STAGES) * 32768;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) umma_f16(tS, desc(qa, kk), desc(kt, kk), IDESC, kk > 0);
        umma_commit(&bar[B_SFULL + X]);
        umma_commit(&bar[B_KEMPTY + j % STAGES]);
      };
      bool ok = wait(B_QFULL, 0, 0x2301) && wait(B_KFULL, 0, 0x2302);
      if (ok) {
        tc_fence_after();
        issue_S(0);
      }
      for (int j = 0; ok && j < nt; ++j) {
        if (!(ok = wait(B_PFULL + X, j & 1, 0x2303))) break;
        if (!(ok = wait(B_VFULL + j % STAGES, (j / STAGES) & 1, 0x2304))) break;
        tc_fence_after();
        const uint32_t vt = vb + (j % STAGES) * 32768;   // O_X += P_X(j) V(j), P from TMEM
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_f16_tmem_a(tO, tS + 64 + 8 * kk, desc(vt, kk), IDESC, (j > 0) || (kk > 0));
        umma_commit(&bar[B_VEMPTY + j % STAGES]);
        if (j + 1 < nt) {
          if (!(ok = wait(B_KFULL + (j + 1) % STAGES, ((j + 1) / STAGES) & 1, 0x2305))) break;
          tc_fence_after();
          issue_S(j + 1);
        } else {
          umma_commit(&bar[B_ODONE + X]);
        }
      }
      // every MMA this thread issued completes before TMEM is released
      umma_commit(&bar[B_DRAIN + X]);
      mbar_wait(&bar[B_DRAIN + X], 0, limit, err, 0x2308);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
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
  const uint8_t* base = static_cast<const uint8_t*>(ws);
  const int smem = f16::Smem::BYTES + 1024;   // > half the SM: one CTA per SM owns all 512 TMEM columns
  cudaError_t e = cudaFuncSetAttribute(fp16_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;   // the setmaxnreg split needs exactly LAUNCH_REGS at launch
  e = cudaFuncGetAttributes(&fa, fp16_attn_kernel);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != f16::LAUNCH_REGS) return cudaErrorInvalidConfiguration;
  const int nt = p.N_pad / TILE;
  fp16_attn_kernel<<<dim3((nt + 1) / 2, p.BH), f16::NUM_THREADS, smem, st>>>(
      p, base + L.qr, base + L.kr, base + L.vt, o, static_cast<WsHeader*>(ws), wait_limit());
  return cudaGetLastError();
}

cudaError_t launch_timeout_probe(void* ws, cudaStream_t st) {
  timeout_probe_kernel<<<1, 32, 0, st>>>(static_cast<WsHeader*>(ws), wait_limit());
  return cudaGetLastError();
}

}  // namespace ra
