// ra_prologue.cu -- the fused prologue of the INT4 path and the FP16 path's
// position encoding.  HBM-bound elementwise work: coalesced 16-byte loads,
// per-element fp32 arithmetic with explicit round-to-nearest intrinsics (no
// FMA contraction, IEEE division) so that codes and scales are reproducible
// bit for bit, warp-shuffle block amax, packed INT4 stores.
//
// RotateAttention (arXiv 2607.02584) review page: 3D RoPE splits head_dim
// into frame/height/width segments (core claim; axiom ledger); the
// RoPE-aware rotation is block-diagonal 2x2 orthogonal, Interleaved on
// adjacent dims (merged into RoPE) or Half, pairing each dim with its
// counterpart in the other half of its segment (Fig. 3 caption); the blocks
// are the 2x2 Hadamard (free-parameter ledger); Q and K are quantised to
// symmetric INT4 per 64-token block, V per channel.
#include <cuda_fp16.h>
#include <cstdint>

#include "ra_internal.h"

namespace ra {
namespace {

constexpr float kRsqrt2 = 0.70710678118654752440f;   // fp32 rounding of 1/sqrt(2)
constexpr float kRsqrt128 = 0.08838834764831844055f; // fp32 rounding of 1/sqrt(128)

struct TokenPos {
  int p[3];
};

__device__ __forceinline__ TokenPos token_pos(const Prob& P, int n) {
  TokenPos t;
  if (n >= P.n_video) {
    t.p[0] = t.p[1] = t.p[2] = 0;   // text tokens: position 0 on every axis (no RoPE)
  } else if (P.fastdiv) {
    const uint32_t u = (uint32_t)n;
    const uint32_t f = P.m_hw ? __umulhi(u, P.m_hw) : u;   // n / (Hh W)
    const uint32_t nw = P.m_w ? __umulhi(u, P.m_w) : u;    // n / W
    t.p[0] = (int)f;
    t.p[1] = (int)(nw - f * (uint32_t)P.Hh);
    t.p[2] = (int)(u - nw * (uint32_t)P.W);
  } else {
    t.p[0] = n / (P.Hh * P.W);
    t.p[1] = (n / P.W) % P.Hh;
    t.p[2] = n % P.W;
  }
  return t;
}

__device__ __forceinline__ int segment_of(const Prob& P, int c) {
  return c < P.off[1] ? 0 : (c < P.off[2] ? 1 : 2);
}

__device__ __forceinline__ void h8_to_f(const uint4& u, float (&f)[8]) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __half22float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Symmetric INT4 code: clamp(rne(v / s), -7, 7) with the IEEE quotient
// fl(v / s); 0 when s == 0.
__device__ __forceinline__ int int4_code(float v, float s) {
  if (s == 0.0f) return 0;
  int q = __float2int_rn(__fdiv_rn(v, s));
  return q > 7 ? 7 : (q < -7 ? -7 : q);
}

// Reciprocal of a scale for int4_codes8: RN(1 / s), or 0 where it would not
// be a finite normal number (s == 0, or s so small or so large that 1 / s
// overflows or is subnormal), which sends the elements to int4_code.
__device__ __forceinline__ float code_recip(float s) {
  const float r = __fdiv_rn(1.0f, s);
  return (r < 3.0e38f && r > 1.0e-37f) ? r : 0.0f;
}

constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23

// Two fp32 products / sums / differences in one instruction, each rounded
// to nearest on its own (bit-identical to two scalar operations).
__device__ __forceinline__ void mul2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// max(a, |b|, |c|) in one three-input instruction
__device__ __forceinline__ float max_abs3(float a, float b, float c) {
  float d;
  asm("{\n\t.reg .f32 ab, ac;\n\tabs.f32 ab, %2;\n\tabs.f32 ac, %3;\n\tmax.f32 %0, %1, ab, ac;\n\t}"
      : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ void sub2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// int4_code(v[e], s[e]) of eight elements without a division per element,
// for |v| <= 7 s (1 + 2^-22) (every element whose amax gave s = fl(amax / 7)),
// as the low byte of t[e] (two's complement; the low nibble is the packed
// code).  With r = RN(1 / s), |v r - v / s| <= |v| 2^-24 / s <= 7.0 * 2^-24
// and |fl(v / s) - v / s| <= 2^-22, so v r is within 6.6e-7 of fl(v / s):
// the two round to the same integer unless v r lies within that of a
// half-integer.  t = v r + 1.5 * 2^23 rounded once is that integer in the low
// mantissa bits (exact: |v r| < 7.5, so no clamp is needed), and
// d = v r - (t - 1.5 * 2^23) tells how close it is to a tie.  If any of the
// eight lies within 1e-5 of a tie, or a scale has no usable reciprocal
// (no_recip), all eight take the IEEE quotient instead.
__device__ __forceinline__ void int4_codes8(const float (&v)[8], const float (&s)[8], const float (&r)[8],
                                            bool no_recip, uint32_t (&t)[8]) {
  float near = no_recip ? 1.0f : 0.0f;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    float t0, t1, u0, u1, d0, d1;
    fma2(t0, t1, v[e], v[e + 1], r[e], r[e + 1], kMagic, kMagic);
    sub2(u0, u1, kMagic, kMagic, t0, t1);
    fma2(d0, d1, v[e], v[e + 1], r[e], r[e + 1], u0, u1);
    near = max_abs3(near, d0, d1);
    t[e] = __float_as_uint(t0);
    t[e + 1] = __float_as_uint(t1);
  }
  if (near > 0.49999f) {
#pragma unroll
    for (int e = 0; e < 8; ++e) t[e] = (uint32_t)int4_code(v[e], s[e]);
  }
}

// Eight codes held in the low bytes of w[0..7] (two's complement) -> one
// word of nibbles, code e in bits 4e .. 4e + 3: the even codes and the odd
// codes gathered bytewise, then interleaved as low and high nibbles.
__device__ __forceinline__ uint32_t pack8_low_nibbles(const uint32_t (&w)[8]) {
  const uint32_t ev = __byte_perm(__byte_perm(w[0], w[2], 0x0040), __byte_perm(w[4], w[6], 0x0040), 0x5410);
  const uint32_t od = __byte_perm(__byte_perm(w[1], w[3], 0x0040), __byte_perm(w[5], w[7], 0x0040), 0x5410);
  return (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
}

__device__ __forceinline__ bool signature_ok(const WsHeader* hdr, const Prob& P, uint32_t site) {
  if (hdr->signature == P.signature) return true;
  if (threadIdx.x == 0) report(const_cast<DeviceErr*>(&hdr->err), DEVERR_WORKSPACE, site);
  return false;
}

// Where a thread's 4 pairs of channels (lo, lo + 1), (lo + 2, lo + 3),
// (hi, hi + 1), (hi + 2, hi + 3) find their table entries:
// entry = base[pp] + pos[axis[pp]] * stride[pp].  Computed once per
// thread with selects on the segment, so that no per-element lookup indexes
// the problem's arrays with a run-time segment (which would put them in
// local memory).
struct PairTab {
  int base[4], stride[4], axis[4];
};

__device__ __forceinline__ int sel3(int s, int a, int b, int c) { return s == 0 ? a : (s == 1 ? b : c); }

__device__ __forceinline__ PairTab pair_tab(const Prob& P, int lo, int hi) {
  PairTab t;
#pragma unroll
  for (int pp = 0; pp < 4; ++pp) {
    const int c = (pp < 2 ? lo : hi) + 2 * (pp & 1);
    const int s = c < P.off[1] ? 0 : (c < P.off[2] ? 1 : 2);
    const int j = (c - sel3(s, P.off[0], P.off[1], P.off[2])) >> 1;
    const int q = sel3(s, P.tab_q[0], P.tab_q[1], P.tab_q[2]);
    t.base[pp] = sel3(s, P.tab_off[0], P.tab_off[1], P.tab_off[2]) + (j & 3) * q + (j >> 2);
    t.stride[pp] = 4 * q;
    t.axis[pp] = s;
  }
  return t;
}

// RoPE of the 4 adjacent pairs held by one thread (channels c0..c0+7 of
// token n).  FORM 0: the RoPE rotation (cos, sin); FORM 1: the Interleaved
// H2 * Rot (alpha, beta); FORM 2: a caller's block times Rot, merged on the
// host (m00, m01, m10, m11).
template <int FORM>
__device__ __forceinline__ void rope8(const PairTab& pt, const float4* __restrict__ tab, const TokenPos& tp,
                                      const float (&x)[8], float (&y)[8], int n_tab, DeviceErr* err) {
#pragma unroll
  for (int pp = 0; pp < 4; ++pp) {
    const int pos = sel3(pt.axis[pp], tp.p[0], tp.p[1], tp.p[2]);
    const int ti = pt.base[pp] + pos * pt.stride[pp];
    float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
    if (in_bounds(ti >= 0 && ti < n_tab, err, 0x101)) {
      if (FORM == 2) {
        t = __ldg(&tab[ti]);
      } else {   // FORM 0 reads (cos, sin), FORM 1 (alpha, beta): one 8-byte load
        const float2 h = __ldg(reinterpret_cast<const float2*>(&tab[ti]) + (FORM == 1 ? 1 : 0));
        if (FORM == 1) { t.z = h.x; t.w = h.y; } else { t.x = h.x; t.y = h.y; }
      }
    }
    const float x0 = x[2 * pp], x1 = x[2 * pp + 1];
    if (FORM == 1) {          // z0 = alpha x0 + beta x1, z1 = beta x0 - alpha x1
      float p0, p1, q0, q1;
      mul2(p0, p1, t.z, t.w, x0, x0);
      mul2(q0, q1, t.w, t.z, x1, x1);
      y[2 * pp] = __fadd_rn(p0, q0);
      y[2 * pp + 1] = __fsub_rn(p1, q1);
    } else if (FORM == 2) {   // z0 = m00 x0 + m01 x1, z1 = m10 x0 + m11 x1
      y[2 * pp] = __fadd_rn(__fmul_rn(t.x, x0), __fmul_rn(t.y, x1));
      y[2 * pp + 1] = __fadd_rn(__fmul_rn(t.z, x0), __fmul_rn(t.w, x1));
    } else {                  // y0 = c x0 - s x1, y1 = s x0 + c x1
      y[2 * pp] = __fsub_rn(__fmul_rn(t.x, x0), __fmul_rn(t.y, x1));
      y[2 * pp + 1] = __fadd_rn(__fmul_rn(t.y, x0), __fmul_rn(t.x, x1));
    }
  }
}

// Normalised 128-point Walsh-Hadamard transform of one row held by 16
// consecutive lanes, 8 channels each (lane g: channels 8g .. 8g + 7): strides
// 1, 2, 4 inside the lane, 8 .. 64 across lanes (lane bit h / 8); the pair
// (k, k + h) becomes (a + b, a - b); then one multiply by fp32(1/sqrt(128)).
// All 32 lanes of the warp must call it together.
__device__ __forceinline__ void hadamard128(float (&z)[8], int g) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (!(e & h)) {
        const float a = z[e], b = z[e + h];
        z[e] = __fadd_rn(a, b);
        z[e + h] = __fsub_rn(a, b);
      }
#pragma unroll
  for (int hl = 1; hl < 16; hl <<= 1) {
    const bool upper = (g & hl) != 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, z[e], hl);
      z[e] = upper ? __fsub_rn(other, z[e]) : __fadd_rn(z[e], other);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) z[e] = __fmul_rn(z[e], kRsqrt128);
}

// Q/K prologue CTA: one 64-token block of one head, QK_THREADS threads; lane
// g = t % 16 holds channels 8g .. 8g + 7 of rows t / 16 + QK_RSTEP i (four
// rows a thread: 64 registers, half the SM's warp slots, against a quarter
// with eight rows).
constexpr int QK_THREADS = 256, QK_RSTEP = QK_THREADS / 16, QK_ROWS = QK_BLOCK / QK_RSTEP;

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < QK_THREADS / 32; ++w) m = fmaxf(m, red[w]);
  return m;
}

// One CTA = one 64-token block of Q or K of one head (QK_THREADS threads).
// Thread t holds 8 channels of rows (t/16) + QK_RSTEP i: channels 8 (t%16) ..
// + 7, or with PAIRS (the Half rotations when every segment and half-segment
// boundary is a multiple of 4) the 4 channels lo .. lo + 3 of the first half
// of a segment and their partners lo + d_s/2 .. + 3, so that the rotation
// needs nothing from other threads.
template <int ROT, bool PAIRS>
__global__ void __launch_bounds__(QK_THREADS, ((ROT == RA_ROT_HALF || ROT == RA_ROT_BLOCKS_HALF) && !PAIRS) ? 3 : 4) qk_quant_kernel(Prob P, const __half* __restrict__ q,
                                                       const __half* __restrict__ k, uint8_t* __restrict__ q4,
                                                       uint8_t* __restrict__ k4, float* __restrict__ sq,
                                                       float* __restrict__ sk, const float4* __restrict__ tab,
                                                       const WsHeader* __restrict__ hdr) {
  __shared__ float red[QK_THREADS / 32];
  constexpr bool HALF_PAIRS = ROT == RA_ROT_HALF || ROT == RA_ROT_BLOCKS_HALF;
  __shared__ float ys[HALF_PAIRS && !PAIRS ? QK_BLOCK : 1][HALF_PAIRS && !PAIRS ? D + 4 : 1];
  DeviceErr* err = const_cast<DeviceErr*>(&hdr->err);
  const int blk = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const __half* x = (which ? k : q) + (size_t)bh * P.N * D;
  uint8_t* out = (which ? k4 : q4) + (size_t)bh * P.N_pad * (D / 2);
  float* scale = (which ? sk : sq) + (size_t)bh * (P.N_pad / QK_BLOCK);
  const int g = threadIdx.x & 15, r0 = threadIdx.x >> 4;   // rows r0 + QK_RSTEP i
  const int c0 = 8 * g;
  int lo = c0, hi = c0 + 4;   // the thread's channels: lo .. lo + 3, hi .. hi + 3
  int seg = 0;                // PAIRS: the segment of lo and hi
  if (PAIRS) {
    // the first half of segment s has split[s] / 8 groups of 4 channels; the
    // 16 threads of a row take them in order (sum over s: 128 / 8 = 16)
    const int q0 = P.split[0] >> 3, q1 = P.split[1] >> 3;
    seg = g < q0 ? 0 : (g < q0 + q1 ? 1 : 2);
    lo = sel3(seg, P.off[0], P.off[1], P.off[2]) + 4 * (g - sel3(seg, 0, q0, q0 + q1));
    hi = lo + (sel3(seg, P.split[0], P.split[1], P.split[2]) >> 1);
  }

  uint4 raw[QK_ROWS];
#pragma unroll
  for (int i = 0; i < QK_ROWS; ++i) {
    const int n = blk * QK_BLOCK + r0 + QK_RSTEP * i;
    const bool ok = n < P.N && in_bounds(bh < P.BH && lo >= 0 && hi + 4 <= D, err, 0x102);
    if (PAIRS) {
      const uint2 a = ok ? __ldg(reinterpret_cast<const uint2*>(x + (size_t)n * D + lo)) : make_uint2(0, 0);
      const uint2 b = ok ? __ldg(reinterpret_cast<const uint2*>(x + (size_t)n * D + hi)) : make_uint2(0, 0);
      raw[i] = make_uint4(a.x, a.y, b.x, b.y);
    } else {
      raw[i] = ok ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)n * D + c0)) : make_uint4(0, 0, 0, 0);
    }
  }
  float z[QK_ROWS][8];
  float amax = 0.0f;
  const PairTab pt = pair_tab(P, lo, hi);
#pragma unroll
  for (int i = 0; i < QK_ROWS; ++i) {
    const int n = blk * QK_BLOCK + r0 + QK_RSTEP * i;
    float xf[8];
    h8_to_f(raw[i], xf);
    const TokenPos tp = token_pos(P, n < P.N ? n : 0);
    rope8<ROT == RA_ROT_INTERLEAVED ? 1 : (ROT == RA_ROT_BLOCKS_INTERLEAVED ? 2 : 0)>(pt, tab, tp, xf, z[i], P.n_tab,
                                                                                      err);
  }
  if (HALF_PAIRS && PAIRS) {
    // pair (o_s + i, o_s + i + d_s/2) = (z[e], z[4 + e]) of the same thread
    float4 r4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {   // block of pair o_s / 2 + i, i = index in the first half
      const int off = sel3(seg, P.off[0], P.off[1], P.off[2]);
      const int bi = (off >> 1) + (lo + e - off);
      r4[e] = ROT == RA_ROT_BLOCKS_HALF && in_bounds(bi >= 0 && bi < D / 2, err, 0x107) ? __ldg(&tab[P.n_tab + bi])
                                                                                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < QK_ROWS; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = z[i][e], b = z[i][4 + e];
        if (ROT == RA_ROT_BLOCKS_HALF) {
          z[i][e] = __fadd_rn(__fmul_rn(r4[e].x, a), __fmul_rn(r4[e].y, b));
          z[i][4 + e] = __fadd_rn(__fmul_rn(r4[e].z, a), __fmul_rn(r4[e].w, b));
        } else {
          z[i][e] = __fmul_rn(__fadd_rn(a, b), kRsqrt2);
          z[i][4 + e] = __fmul_rn(__fsub_rn(a, b), kRsqrt2);
        }
      }
  } else if (HALF_PAIRS) {
    // pair (o_s + i, o_s + i + d_s/2): each thread has its own channel in a
    // register and reads the partner's value of the same row from shared memory
#pragma unroll
    for (int i = 0; i < QK_ROWS; ++i) {
      float4* row = reinterpret_cast<float4*>(&ys[r0 + QK_RSTEP * i][c0]);
      row[0] = make_float4(z[i][0], z[i][1], z[i][2], z[i][3]);
      row[1] = make_float4(z[i][4], z[i][5], z[i][6], z[i][7]);
    }
    __syncthreads();
    auto pair_rot = [](bool first, float self, float other, const float4& r4) {
      const float a = first ? self : other, b = first ? other : self;
      if (ROT == RA_ROT_BLOCKS_HALF)
        return first ? __fadd_rn(__fmul_rn(r4.x, a), __fmul_rn(r4.y, b))
                     : __fadd_rn(__fmul_rn(r4.z, a), __fmul_rn(r4.w, b));
      return first ? __fmul_rn(__fadd_rn(a, b), kRsqrt2) : __fmul_rn(__fsub_rn(a, b), kRsqrt2);
    };
    // (the PAIRS instance serves the layouts with every boundary a multiple of 4)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int c = c0 + e;
      const int s = segment_of(P, c);
      const int h = sel3(s, P.split[0], P.split[1], P.split[2]) >> 1;
      const int off = sel3(s, P.off[0], P.off[1], P.off[2]);
      const bool first = (c - off) < h;
      const int pc = first ? c + h : c - h;
      const float4 r4 = ROT == RA_ROT_BLOCKS_HALF &&
                                in_bounds((off >> 1) + (c - off) - (first ? 0 : h) < D / 2, err, 0x104)
                            ? __ldg(&tab[P.n_tab + (off >> 1) + (c - off) - (first ? 0 : h)])
                                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < QK_ROWS; ++i) z[i][e] = pair_rot(first, z[i][e], ys[r0 + QK_RSTEP * i][pc], r4);
    }
  }
  if (ROT == RA_ROT_FULL) {
#pragma unroll
    for (int i = 0; i < QK_ROWS; ++i) hadamard128(z[i], g);
  }
#pragma unroll
  for (int i = 0; i < QK_ROWS; ++i)
#pragma unroll
    for (int e = 0; e < 8; e += 2) amax = max_abs3(amax, z[i][e], z[i][e + 1]);
  amax = block_max(amax, red);
  // the workspace's tables were read above (in bounds whatever they hold);
  // nothing is written unless they are this problem's
  if (!signature_ok(hdr, P, 0x100)) return;
  const float s = __fdiv_rn(amax, 7.0f);
  const float rs = code_recip(s);
  // codes of each row: one IEEE division per block for the scale and its
  // reciprocal, none per element (int4_codes8)
  float s8[8], r8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    s8[e] = s;
    r8[e] = rs;
  }
#pragma unroll
  for (int i = 0; i < QK_ROWS; ++i) {
    uint32_t tb[8];
    int4_codes8(z[i], s8, r8, rs == 0.0f, tb);
    const int n = blk * QK_BLOCK + r0 + QK_RSTEP * i;
    if (in_bounds(n < P.N_pad && bh < P.BH, err, 0x105)) {
      const uint32_t w = pack8_low_nibbles(tb);   // codes of lo .. lo + 3 low, hi .. hi + 3 high
      if (PAIRS) {
        *reinterpret_cast<uint16_t*>(out + (size_t)n * (D / 2) + lo / 2) = (uint16_t)(w & 0xFFFFu);
        *reinterpret_cast<uint16_t*>(out + (size_t)n * (D / 2) + hi / 2) = (uint16_t)(w >> 16);
      } else {
        *reinterpret_cast<uint32_t*>(out + (size_t)n * (D / 2) + 4 * g) = w;
      }
    }
  }
  if (threadIdx.x == 0 && in_bounds(blk < P.N_pad / QK_BLOCK && bh < P.BH, err, 0x106)) scale[blk] = s;
}

// Per-(head, channel) amax of V over a 256-token chunk, merged with
// atomicMax on the bit pattern (valid for non-negative floats).
__global__ void __launch_bounds__(128) v_amax_kernel(Prob P, const __half* __restrict__ v,
                                                     uint32_t* __restrict__ vamax,
                                                     const WsHeader* __restrict__ hdr) {
  __shared__ float part[8][D];
  if (!signature_ok(hdr, P, 0x200)) return;
  DeviceErr* err = const_cast<DeviceErr*>(&hdr->err);
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int g = threadIdx.x & 15, r0 = threadIdx.x >> 4;
  const __half* x = v + (size_t)bh * P.N * D;
  float m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  // rows past N count as zero rows; every lane runs every iteration, so the
  // Hadamard's shuffles always see the whole warp
  const int rows = min(256, P.N - chunk * 256);
  const int iters = P.v_rot ? 32 : (rows + 7) / 8;
  for (int i = 0; i < iters; ++i) {
    const int n = chunk * 256 + r0 + 8 * i;
    float f[8];
    if (n < P.N && in_bounds(bh < P.BH, err, 0x201)) {
      h8_to_f(__ldg(reinterpret_cast<const uint4*>(x + (size_t)n * D + 8 * g)), f);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = 0.0f;
    }
    if (P.v_rot) hadamard128(f, g);
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(f[e]));
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[r0][8 * g + e] = m[e];
  __syncthreads();
  const int c = threadIdx.x;
  float r = part[0][c];
#pragma unroll
  for (int i = 1; i < 8; ++i) r = fmaxf(r, part[i][c]);
  if (in_bounds(bh < P.BH, err, 0x202)) atomicMax(&vamax[(size_t)bh * D + c], __float_as_uint(r));
}

// 8 x 8 transpose of nibbles: on entry r[i] holds nibble e of row i in bits
// 4e .. 4e + 3; on return r[e] holds nibble i of the old r[i] in bits 4i ..
// 4i + 3.  Three block swaps: 4 x 4 blocks (16-bit halves), 2 x 2 blocks
// (bytes), single nibbles.
__device__ __forceinline__ void transpose8_nibbles(uint32_t (&r)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t a = r[i], b = r[i + 4];
    r[i] = __byte_perm(a, b, 0x5410);
    r[i + 4] = __byte_perm(a, b, 0x7632);
  }
#pragma unroll
  for (int i = 0; i < 8; i += (i & 1) ? 3 : 1) {   // 0, 1, 4, 5
    const uint32_t a = r[i], b = r[i + 2];
    r[i] = __byte_perm(a, b, 0x6240);
    r[i + 2] = __byte_perm(a, b, 0x7351);
  }
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const uint32_t a = r[i], b = r[i + 1];
    r[i] = (a & 0x0F0F0F0Fu) | ((b << 4) & 0xF0F0F0F0u);
    r[i + 1] = ((a >> 4) & 0x0F0F0F0Fu) | (b & 0xF0F0F0F0u);
  }
}

// Sum of the eight signed nibbles (two's complement) of w, plus 64: x ^ 8
// maps a nibble s in [-8, 7] to s + 8 in [0, 15]; the bytes of the even and
// of the odd nibbles are summed by dp4a onto acc.
__device__ __forceinline__ int nibble_sum_plus64(uint32_t w, int acc) {
  const uint32_t x = w ^ 0x88888888u;
  acc = __dp4a((int)(x & 0x0F0F0F0Fu), 0x01010101, acc);
  return __dp4a((int)((x >> 4) & 0x0F0F0F0Fu), 0x01010101, acc);
}

// One CTA = one 64-token block of V of one head: codes with the per-channel
// scale, transposed packing (channel-major, two tokens per byte) and the
// block's column sums.  Thread t holds channels 8 (t % 16) .. + 7 of the 8
// consecutive tokens 8 (t / 16) .. + 7: it packs each token's 8 codes into a
// word, transposes the 8 x 8 nibbles in registers (one word per channel, its
// 8 tokens in order), and the words meet in shared memory, one 32-byte row of
// 64 tokens per channel.  The 8 row loads are issued first, before the
// workspace signature is read, and the channel scales are computed once per
// channel (thread c: channel c) and shared; 8 CTAs per SM (64 registers).
__global__ void __launch_bounds__(128, 8) v_quant_kernel(Prob P, const __half* __restrict__ v,
                                                      const uint32_t* __restrict__ vamax,
                                                      uint8_t* __restrict__ v4t, float* __restrict__ sv,
                                                      int32_t* __restrict__ vsum,
                                                      const WsHeader* __restrict__ hdr) {
  __shared__ __align__(16) uint32_t words[8][D];   // [token group][channel]
  __shared__ __align__(16) float scl[2][D];         // per channel: s, RN(1 / s)
  DeviceErr* err = const_cast<DeviceErr*>(&hdr->err);
  const int blk = blockIdx.x, bh = blockIdx.y;
  const int g = threadIdx.x & 15, r0 = threadIdx.x >> 4;
  const __half* x = v + (size_t)bh * P.N * D;
  uint4 raw[8];   // token 8 r0 + i, channels 8 g .. 8 g + 7
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int n = blk * QK_BLOCK + 8 * r0 + i;
    raw[i] = n < P.N && in_bounds(bh < P.BH, err, 0x301) ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)n * D + 8 * g))
                                                         : make_uint4(0, 0, 0, 0);
  }
  {   // one division pair per channel: thread c computes channel c's
    const int c = threadIdx.x;
    const float sc = __fdiv_rn(__uint_as_float(vamax[(size_t)bh * D + c]), 7.0f);
    scl[0][c] = sc;
    scl[1][c] = code_recip(sc);
    if (!signature_ok(hdr, P, 0x300)) return;
    if (blk == 0) sv[(size_t)bh * D + c] = sc;
  }
  __syncthreads();
  float s[8], rs[8];
  {
    const float4* s4 = reinterpret_cast<const float4*>(&scl[0][8 * g]);
    const float4* r4 = reinterpret_cast<const float4*>(&scl[1][8 * g]);
    const float4 sa = s4[0], sb = s4[1], ra = r4[0], rb = r4[1];
    s[0] = sa.x; s[1] = sa.y; s[2] = sa.z; s[3] = sa.w; s[4] = sb.x; s[5] = sb.y; s[6] = sb.z; s[7] = sb.w;
    rs[0] = ra.x; rs[1] = ra.y; rs[2] = ra.z; rs[3] = ra.w; rs[4] = rb.x; rs[5] = rb.y; rs[6] = rb.z; rs[7] = rb.w;
  }
  bool no_recip = false;
#pragma unroll
  for (int e = 0; e < 8; ++e) no_recip |= rs[e] == 0.0f;
  uint32_t tw[8];   // token 8 r0 + i: its 8 codes as nibbles
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float f[8];
    h8_to_f(raw[i], f);
    if (P.v_rot) hadamard128(f, g);
    uint32_t tb[8];
    int4_codes8(f, s, rs, no_recip, tb);
    tw[i] = pack8_low_nibbles(tb);
  }
  transpose8_nibbles(tw);   // tw[e]: channel 8 g + e, tokens 8 r0 .. 8 r0 + 7
  uint4* wrow = reinterpret_cast<uint4*>(&words[r0][8 * g]);
  wrow[0] = make_uint4(tw[0], tw[1], tw[2], tw[3]);
  wrow[1] = make_uint4(tw[4], tw[5], tw[6], tw[7]);
  __syncthreads();
  const int c = threadIdx.x;
  uint32_t w[8];
  int sum = -512;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    w[t] = words[t][c];
    sum = nibble_sum_plus64(w[t], sum);
  }
  // tile-major V^T: [bh][tile][channel][64 bytes], this block is half (blk % 2) of tile blk / 2
  uint4* dst = reinterpret_cast<uint4*>(v4t + (((size_t)bh * (P.N_pad / TILE) + blk / 2) * D + c) * (TILE / 2) +
                                        (size_t)(blk % 2) * (QK_BLOCK / 2));
  if (!in_bounds(bh < P.BH && blk < P.N_pad / QK_BLOCK, err, 0x302)) return;
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  vsum[((size_t)bh * (P.N_pad / QK_BLOCK) + blk) * D + c] = sum;
}

// FP16 path: RoPE of Q and K rounded to fp16 ([BH][N_pad][128], padded rows
// zero) and V transposed to [BH][128][N_pad] fp16 (padded tokens zero).
__global__ void __launch_bounds__(128) fp16_prologue_kernel(Prob P, const __half* __restrict__ q,
                                                            const __half* __restrict__ k,
                                                            const __half* __restrict__ v, __half* __restrict__ qr,
                                                            __half* __restrict__ kr, __half* __restrict__ vt,
                                                            const float4* __restrict__ tab,
                                                            const WsHeader* __restrict__ hdr) {
  __shared__ __half tr[QK_BLOCK][D + 8];
  if (!signature_ok(hdr, P, 0x400)) return;
  DeviceErr* err = const_cast<DeviceErr*>(&hdr->err);
  const int blk = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  if (!in_bounds(bh < P.BH && blk < P.N_pad / QK_BLOCK, err, 0x401)) return;
  const int g = threadIdx.x & 15, r0 = threadIdx.x >> 4;
  const int c0 = 8 * g;
  const int nt = P.N_pad / TILE;
  const __half* x = (which == 0 ? q : which == 1 ? k : v) + (size_t)bh * P.N * D;
  if (which < 2) {
    // operand image: tile n / 128 is 32 KB, channels 0..63 and 64..127 in two
    // 128-byte-swizzled K-major atoms of 16 KB
    uint8_t* img = reinterpret_cast<uint8_t*>(which == 0 ? qr : kr) + (size_t)bh * nt * 32768;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int n = blk * QK_BLOCK + r0 + 8 * i;
      uint4 o = make_uint4(0, 0, 0, 0);
      if (n < P.N) {
        float xf[8], y[8];
        h8_to_f(__ldg(reinterpret_cast<const uint4*>(x + (size_t)n * D + c0)), xf);
        rope8<0>(pair_tab(P, c0, c0 + 4), tab, token_pos(P, n), xf, y, P.n_tab, err);
        __half2* h = reinterpret_cast<__half2*>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = __floats2half2_rn(y[2 * e], y[2 * e + 1]);
      }
      *reinterpret_cast<uint4*>(img + (size_t)(n / TILE) * 32768 + (c0 >> 6) * 16384 +
                                sw128_off(n % TILE, (c0 & 63) >> 3)) = o;
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + 8 * i, n = blk * QK_BLOCK + r;
    uint4 u = n < P.N ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)n * D + c0)) : make_uint4(0, 0, 0, 0);
    const __half* h = reinterpret_cast<const __half*>(&u);
#pragma unroll
    for (int e = 0; e < 8; ++e) tr[r][c0 + e] = h[e];
  }
  __syncthreads();
  // thread c writes channel c's 64 tokens (128 bytes) of this block: row c
  // of the V^T operand image of key tile blk / 2, atom blk % 2
  const int c = threadIdx.x;
  uint8_t* dst = reinterpret_cast<uint8_t*>(vt) + ((size_t)bh * nt + blk / 2) * 32768 + (blk & 1) * 16384;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    uint4 o;
    __half* h = reinterpret_cast<__half*>(&o);
#pragma unroll
    for (int e = 0; e < 8; ++e) h[e] = tr[8 * t + e][c];
    *reinterpret_cast<uint4*>(dst + sw128_off(c, t)) = o;
  }
}

}  // namespace

cudaError_t launch_prologue(const Prob& p, const __half* q, const __half* k, const __half* v, uint8_t* q4,
                            uint8_t* k4, uint8_t* v4t, float* sq, float* sk, float* sv, int32_t* vsum, void* ws,
                            cudaStream_t st) {
  const WsLayout L = ws_layout(p);
  char* base = static_cast<char*>(ws);
  const WsHeader* hdr = reinterpret_cast<const WsHeader*>(base);
  const float4* tab = reinterpret_cast<const float4*>(base + L.tables);
  uint32_t* vamax = reinterpret_cast<uint32_t*>(base + L.vamax);
  const dim3 gqk(p.N_pad / QK_BLOCK, p.BH, 2);
#define RA_QK(ROT, PAIRS) qk_quant_kernel<ROT, PAIRS><<<gqk, QK_THREADS, 0, st>>>(p, q, k, q4, k4, sq, sk, tab, hdr)
  switch (p.rot) {
    case RA_ROT_NONE: RA_QK(RA_ROT_NONE, false); break;
    case RA_ROT_INTERLEAVED: RA_QK(RA_ROT_INTERLEAVED, false); break;
    case RA_ROT_FULL: RA_QK(RA_ROT_FULL, false); break;
    case RA_ROT_BLOCKS_INTERLEAVED: RA_QK(RA_ROT_BLOCKS_INTERLEAVED, false); break;
    case RA_ROT_BLOCKS_HALF:
      if (p.half4) RA_QK(RA_ROT_BLOCKS_HALF, true);
      else RA_QK(RA_ROT_BLOCKS_HALF, false);
      break;
    default:
      if (p.half4) RA_QK(RA_ROT_HALF, true);
      else RA_QK(RA_ROT_HALF, false);
      break;
  }
#undef RA_QK
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(vamax, 0, sizeof(uint32_t) * (size_t)p.BH * D, st);
  if (e != cudaSuccess) return e;
  v_amax_kernel<<<dim3((p.N + 255) / 256, p.BH), 128, 0, st>>>(p, v, vamax, hdr);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  v_quant_kernel<<<dim3(p.N_pad / QK_BLOCK, p.BH), 128, 0, st>>>(p, v, vamax, v4t, sv, vsum, hdr);
  return cudaGetLastError();
}

cudaError_t launch_fp16_prologue(const Prob& p, const __half* q, const __half* k, const __half* v, void* ws,
                                 cudaStream_t st) {
  const WsLayout L = ws_layout(p);
  char* base = static_cast<char*>(ws);
  fp16_prologue_kernel<<<dim3(p.N_pad / QK_BLOCK, p.BH, 3), 128, 0, st>>>(
      p, q, k, v, reinterpret_cast<__half*>(base + L.qr), reinterpret_cast<__half*>(base + L.kr),
      reinterpret_cast<__half*>(base + L.vt), reinterpret_cast<const float4*>(base + L.tables),
      reinterpret_cast<const WsHeader*>(base));
  return cudaGetLastError();
}

}  // namespace ra
