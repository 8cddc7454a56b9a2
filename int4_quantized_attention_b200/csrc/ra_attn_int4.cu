// ra_attn_int4.cu -- INT4 attention forward, warp-specialised, on the sm_100a
// 5th-generation tensor cores.
//
// RotateAttention (arXiv 2607.02584) review page: INT4 FlashAttention with
// online softmax (abstract); range-optimised P quantisation -- P = exp(s - m)
// in [0, 1] mapped to rne(15 P) - 8 in [-8, 7], fixed scale 15, zero-point -8
// (Sec. 4.2 as summarised by the referee report; free-parameter ledger) --
// with the zero-point corrected through the V column sums.
//
// One CTA = one (batch*head, pair of 128-row query tiles A and B); 384
// threads in three warpgroups:
//   WG0 (warps 0-3)    softmax of tile A, thread t = query row t = TMEM lane t
//   WG1 (warps 4-7)    softmax of tile B
//   WG2 warp 8         bulk-copy producer: the two Q operand tiles once, then
//                      the K and V^T operand tiles (16 KB each) into a
//                      3-stage ring
//       warps 9, 10    MMA issuers, one thread per query tile (warp 9 also
//                      owns the TMEM allocation)
//       warp 11        idle after set-up
// The packed INT4 inputs are expanded once per call, by expand_kernel, into
// INT8 operand images laid out exactly as the MMAs read them from SMEM, so
// the attention kernel itself only copies tiles.
//
// TMEM (512 columns): S_A | S_B | O_A | O_B, 128 int32 columns each.  The P
// operand (128 rows x 128 u8 = 16 KB) goes to SMEM, double-buffered per
// query tile, laid out like a Q tile.  So the S columns are free as soon as
// the softmax warps hold S in registers: tile X's thread issues S_X(j+1)
// right then, and S_X(j+1) is ready when the softmax finishes tile j; it
// issues O_X += W_X(j) V(j) once the four softmax warps have stored W_X(j).
// The two tiles' threads share the tensor core and the operand ring, which
// is refilled once both have consumed a stage.
//
// A row whose running max moves has its int32 accumulator rescaled in TMEM by
// its own softmax thread, after P.V(j-1) has landed (issued a whole tile
// earlier) and before it releases W(j).
//
// S_X(j) is the int32 256 S of the four integer MMAs (the first one starts
// the accumulator).  The softmax takes the row max on the integers and
// converts to fp32 (exact: |256 S| < 2^24) only what it exponentiates.
//
// The P operand is w = rne(15 * 2^(x - m)) = code + 8 in [0, 15] (with the
// symmetric P map instead: w = rne(7 * 2^(x - m)) = code), fed as an
// unsigned 8-bit operand: the tensor core then sums (code + 8) * v, which is
// sum code * v + 8 * colsum(v) -- the zero-point correction, bit-identical.
// The int32 P.V accumulator stays in TMEM across tiles; the rescale rounds
// acc * exp2(m_old - m_new) back to an integer (rows whose max did not move
// keep theirs).  The normaliser l is the running sum of w.
//
// INT4 codes are expanded to 16*code (the nibble placed in the high half of
// the byte), so S comes out as 256*S and P.V as 16*P.V, exactly; both factors
// fold into the dequantisation.  Within every 8-element group the expanded
// operands hold even elements first, then odd ones (channels for Q and K,
// keys for V^T); the P operand is packed in the same key order.
//
// Keys past N (the ragged last tile) hold zero K and V codes: their P.V
// contribution is zero whatever their w, so only the max and the normaliser
// must exclude them; their P bytes are zeroed as well.
#include <cuda_fp16.h>
#include <cstdint>

#include "ra_internal.h"

namespace ra {
namespace {

constexpr int NUM_THREADS = 384;
#ifndef RA_OP_STAGES
#define RA_OP_STAGES 3
#endif
constexpr int OP_STAGES = RA_OP_STAGES;   // INT8 K / V^T operand tiles (bulk copies)
// Register split: launched at LAUNCH_REGS per thread (384 x 168 = 64512);
// the copy/MMA warpgroup drops to ISSUE_REGS, the two softmax warpgroups
// rise to SOFTMAX_REGS: 256 x 216 + 128 x 72 = 64512.  (With 208 the softmax
// loop kept a few values in local memory; 216 runs 2-4 % faster.)
constexpr int LAUNCH_REGS = 168, SOFTMAX_REGS = 216, ISSUE_REGS = 72;
static_assert(256 * SOFTMAX_REGS + 128 * ISSUE_REGS <= NUM_THREADS * LAUNCH_REGS, "register split");

constexpr uint32_t IDESC_QK = make_idesc(2, 1, 1, 128, 128);   // s32 += s8 x s8
constexpr uint32_t IDESC_PV = make_idesc(2, 0, 1, 128, 128);   // s32 += u8 x s8
constexpr float LOG2E = 1.4426950408889634f;
constexpr float SQRT_D = 11.313708498984761f;
constexpr float MAGIC = 12582912.0f;                           // 1.5 * 2^23
constexpr int MAGIC_BITS = 0x4B400000;
constexpr int S_PAD = -4000000;   // below any 256*S (|256 S| <= 1.6e6)

// max of three int32 (two compares)
__device__ __forceinline__ int imax3(int a, int b, int c) { return max(max(a, b), c); }

struct Smem {
  static constexpr uint32_t QA = 0, QB = 16384;   // INT8 Q operand tiles
  static constexpr uint32_t OP = 32768;           // OP_STAGES x 32 KB: INT8 K (+0), V^T (+16 KB)
  static constexpr uint32_t P = OP + OP_STAGES * 32768;   // [tile][j % 2] 16 KB u8 P operands, laid out like Q
  static constexpr uint32_t BAR = P + 65536;
  static constexpr uint32_t BYTES = BAR + 512;
};
static_assert(Smem::BYTES + 1024 <= 232448, "shared memory per CTA");

// P_FULL[tile][b] and PV_DONE[tile][b] serve the KV tiles j with j % 2 == b:
// a softmax warp may store P(j+1) while another still works on P(j).
enum : int {
  B_OP_FULL = 0, B_OP_EMPTY = OP_STAGES, B_QFULL = 2 * OP_STAGES, B_S_FULL = B_QFULL + 1, B_S_EMPTY = B_S_FULL + 2,
  B_P_FULL = B_S_EMPTY + 2, B_PV_DONE = B_P_FULL + 4, B_DRAIN = B_PV_DONE + 4, NBAR = B_DRAIN + 2
};
static_assert(8 * NBAR + 8 <= 512, "barrier area");

// 4 packed words (32 codes) -> two 16-byte chunks of 16*code, evens then odds
// per 8-element group.
__device__ __forceinline__ void widen16(const uint4 u, uint4& a, uint4& b) {
  a = make_uint4((u.x << 4) & 0xF0F0F0F0u, u.x & 0xF0F0F0F0u, (u.y << 4) & 0xF0F0F0F0u, u.y & 0xF0F0F0F0u);
  b = make_uint4((u.z << 4) & 0xF0F0F0F0u, u.z & 0xF0F0F0F0u, (u.w << 4) & 0xF0F0F0F0u, u.w & 0xF0F0F0F0u);
}

// All 128 columns of this warp's 32 lanes in one load.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
               : "r"(taddr));
}

// P word k (0..31) holds, in byte b, key 8 (k / 2) + 2 b + (k % 2).  Byte mask
// of the keys < nvalid.
__device__ __forceinline__ uint32_t p_word_mask(int k, int nvalid) {
  uint32_t m = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const int key = 8 * (k >> 1) + 2 * b + (k & 1);
    m |= (key < nvalid ? 0xFFu : 0u) << (8 * b);
  }
  return m;
}

// INT4 -> INT8 operand images: one thread per 16 packed bytes (32 codes of
// one row).  Q and K rows are tokens, V^T rows are channels (its tiles are
// already 128 keys wide); row r of 128-row tile t lands, as 16 * code with
// even then odd elements of every 8-group, 128-byte swizzled at
// image + (b*H + h, t) * 16 KB.  The image of a tile is the SMEM operand of
// the MMA byte for byte.
__global__ void __launch_bounds__(256) expand_kernel(const uint8_t* __restrict__ q4, const uint8_t* __restrict__ k4,
                                                     const uint8_t* __restrict__ v4t, uint8_t* __restrict__ qimg,
                                                     uint8_t* __restrict__ kimg, uint8_t* __restrict__ vimg,
                                                     size_t units, DeviceErr* err) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= units) return;
  // units = packed bytes / 16 (4 per 128-byte image row, 512 per 16 KB tile);
  // the images hold 32 bytes per unit
  if (!in_bounds((i >> 9) * 16384 + 16384 <= units * 32, err, 0x4001)) return;
  const int which = blockIdx.y;
  const uint8_t* src = which == 0 ? q4 : (which == 1 ? k4 : v4t);
  uint8_t* dst = which == 0 ? qimg : (which == 1 ? kimg : vimg);
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(src) + i);
  const size_t grow = i >> 2;   // (b*H + h) * N_pad + 128 t + r
  const uint32_t h = (uint32_t)(i & 3), r = (uint32_t)(grow & 127);
  uint8_t* tile = dst + (grow >> 7) * 16384;
  uint4 c0, c1;
  widen16(u, c0, c1);
  *reinterpret_cast<uint4*>(tile + sw128_off(r, 2 * h)) = c0;
  *reinterpret_cast<uint4*>(tile + sw128_off(r, 2 * h + 1)) = c1;
}

struct KernelArgs {
  Prob P;
  const uint8_t* qimg;   // INT8 operand images [BH][N_pad / 128][16 KB]
  const uint8_t* kimg;
  const uint8_t* vimg;
  const float* sq;
  const float* sk;
  const float* sv;
  __half* o;
  WsHeader* hdr;
  uint64_t limit;
  int dbg_bh, dbg_qt, dbg_kv;
  int32_t* dbg_s;
  int8_t* dbg_p;
};

// DBG: the test-only instance that runs one CTA at the given tiles and
// exports one S tile and its P codes; the production instance carries none
// of that code.
template <bool DBG>
__global__ void __launch_bounds__(NUM_THREADS, 1) int4_attn_kernel(const KernelArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Smem::BAR);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Smem::BAR + 8 * NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Smem::BAR + 8 * NBAR + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Prob& P = a.P;
  constexpr bool dbg_run = DBG;
  const int n_qt = P.N_pad / TILE, nt = n_qt, nblk = P.N_pad / QK_BLOCK;
  const int qt0 = 2 * (blockIdx.x + (dbg_run ? a.dbg_qt / 2 : 0));
  const int bh = blockIdx.y + (dbg_run ? a.dbg_bh : 0);
  const bool hasB = qt0 + 1 < n_qt;
  DeviceErr* err = &a.hdr->err;
  const uint64_t limit = a.limit;
  // the grid covers the problem exactly: every index below derives from qt0
  // (< n_qt), bh (< BH) and the KV tile j (< nt)
  if (!in_bounds(qt0 < n_qt && bh < P.BH, err, 0x4010)) return;

  if (tid == 0) {
    for (int i = 0; i < OP_STAGES; ++i) {
      mbar_init(&bar[B_OP_FULL + i], 1);
      mbar_init(&bar[B_OP_EMPTY + i], hasB ? 2 : 1);   // one commit per query tile's MMA thread
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[B_S_FULL + i], 1);
      mbar_init(&bar[B_S_EMPTY + i], 4);  // the softmax warps have S in registers
      mbar_init(&bar[B_P_FULL + 2 * i], 4);
      mbar_init(&bar[B_P_FULL + 2 * i + 1], 4);
      mbar_init(&bar[B_PV_DONE + 2 * i], 1);
      mbar_init(&bar[B_PV_DONE + 2 * i + 1], 1);
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
      const uint32_t row = tid & 127;
      auto wait_all = [&](int b, uint32_t parity, uint32_t site) {
        return __all_sync(0xffffffffu, mbar_wait_abortable(&bar[b], parity, abort_flag, limit, err, site));
      };
      bool ok = true;
      {
        const int grow = (qt0 + X) * TILE + (int)row;
        const float kq = in_bounds(grow / QK_BLOCK < nblk, err, 0x4011)
                             ? __fmul_rn(a.sq[(size_t)bh * nblk + grow / QK_BLOCK], LOG2E / (SQRT_D * 256.0f))
                             : 0.0f;
        // P map: w = rne(pscale * P); range-optimised: pscale 15, code = w - 8;
        // symmetric: pscale 7, code = w.  w = 0 wherever pscale * 2^x <= 1/2,
        // i.e. x <= log2(1 / (2 pscale)) (-4.91 and -3.81): skip_below lies under it.
        const float pscale = P.p_mode == RA_P_SYMMETRIC ? 7.0f : 15.0f;
        const float skip_below = P.p_mode == RA_P_SYMMETRIC ? -4.0f : -5.0f;
        const int zp = P.p_mode == RA_P_SYMMETRIC ? 0 : 8;
        const float* skb = a.sk + (size_t)bh * nblk;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tbase + X * 128 + lane_off, tO = tbase + 256 + X * 128 + lane_off;
        const bool dbg_tile = dbg_run && (qt0 + X) == a.dbg_qt;
        const int tail = P.N - (nt - 1) * TILE;   // valid keys in the last tile, 1..128
        float m = -INFINITY, l = 0.0f;
        bool zbuf0 = false, zbuf1 = false;   // this warp's rows of P buffer 0 / 1 hold zeros
        float skn0 = __ldg(skb), skn1 = __ldg(skb + 1);
        {   // O starts at MB (the bits of 1.5 * 2^23); the P.V MMAs add integers to it
          uint32_t mb[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) mb[e] = (uint32_t)MAGIC_BITS;
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_st32(tO + 32 * c, mb);
          tmem_wait_st();
        }
        for (int j = 0; j < nt; ++j) {
          const float sk0 = skn0, sk1 = skn1;
          if (j + 1 < nt && in_bounds(2 * j + 3 < nblk, err, 0x4012)) {   // next tile's K scales, a tile ahead
            skn0 = __ldg(skb + 2 * j + 2);
            skn1 = __ldg(skb + 2 * j + 3);
          }
          if (!(ok = wait_all(B_S_FULL + X, j & 1, 0x4102))) break;
          tc_fence_after();
          uint32_t s[128];
          tmem_ld128(tS, s);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_S_EMPTY + X]);   // S_X(j+1) may overwrite the S columns
          const int nvalid = (j == nt - 1) ? tail : TILE;
          if (dbg_tile && j == a.dbg_kv) {   // S = (256 S) >> 8, exactly
#pragma unroll
            for (int n = 0; n < 128; ++n) a.dbg_s[row * TILE + n] = n < nvalid ? ((int)s[n] >> 8) : 0;
          }
          if (nvalid < TILE) {
#pragma unroll
            for (int n = 0; n < 128; ++n)
              if (n >= nvalid) s[n] = (uint32_t)S_PAD;
          }
          const float c0 = __fmul_rn(kq, sk0), c1 = __fmul_rn(kq, sk1);
          // row max of the int32 256 S of each 64-key half, then as floats
          // (exact: |256 S| < 2^24)
          int mh[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            mh[c] = imax3((int)s[16 * c], (int)s[16 * c + 1], (int)s[16 * c + 2]);
#pragma unroll
            for (int n = 3; n < 15; n += 2) mh[c] = imax3(mh[c], (int)s[16 * c + n], (int)s[16 * c + n + 1]);
            mh[c] = max(mh[c], (int)s[16 * c + 15]);
          }
          const float mx0 = __int2float_rn(max(imax3(mh[0], mh[1], mh[2]), mh[3]));
          const float mx1 = __int2float_rn(max(imax3(mh[4], mh[5], mh[6]), mh[7]));
          float tmax = __fmul_rn(mx0, c0);
          if (nvalid > 64) tmax = fmaxf(tmax, __fmul_rn(mx1, c1));
          const float m_new = fmaxf(m, tmax);
          const bool moved = j > 0 && m_new > m;
          const float alpha = moved ? ex2(m - m_new) : 1.0f;
          m = m_new;
          const float negm = -m;
          // w = 0 exactly wherever 15 * 2^x <= 1/2; x is monotone in S, so a
          // 64-key half whose largest x is below -5 holds only zero codes.
          // Skip its exponentials when that is so for every row of the warp.
          const bool zero_half[2] = {__all_sync(0xffffffffu, fmaf(mx0, c0, negm) < skip_below) != 0,
                                     __all_sync(0xffffffffu, fmaf(mx1, c1, negm) < skip_below) != 0};
          uint32_t L = 0;
          uint32_t pw[32];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (zero_half[h]) {
#pragma unroll
              for (int k = 16 * h; k < 16 * h + 16; ++k) pw[k] = 0u;
              continue;
            }
#pragma unroll
            for (int k = 16 * h; k < 16 * h + 16; k += 2) {   // 8 keys per pair of words: evens, then odds
              uint32_t wb[8];
              const float ch = h ? c1 : c0;
#pragma unroll
              for (int e = 0; e < 8; e += 2) {   // x = 256 S c - m, w = rne(pscale 2^x): pairs
                const int n = 4 * k + e;
                float x0, x1, w0, w1;
                fma2(x0, x1, __int2float_rn((int)s[n]), __int2float_rn((int)s[n + 1]), ch, ch, negm, negm);
                fma2(w0, w1, pscale, pscale, ex2(x0), ex2(x1), MAGIC, MAGIC);   // low byte = w
                wb[e] = __float_as_uint(w0);
                wb[e + 1] = __float_as_uint(w1);
              }
              const uint32_t e02 = __byte_perm(wb[0], wb[2], 0x0040), e46 = __byte_perm(wb[4], wb[6], 0x0040);
              const uint32_t o13 = __byte_perm(wb[1], wb[3], 0x0040), o57 = __byte_perm(wb[5], wb[7], 0x0040);
              pw[k] = __byte_perm(e02, e46, 0x5410);
              pw[k + 1] = __byte_perm(o13, o57, 0x5410);
              L = __dp4a(pw[k], 0x01010101u, L);
              L = __dp4a(pw[k + 1], 0x01010101u, L);
            }
          }
          if (nvalid < TILE) {   // keys past N leave the normaliser and the operand
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const uint32_t keep = p_word_mask(k, nvalid);
              L -= __dp4a(pw[k] & ~keep, 0x01010101u, 0u);
              pw[k] &= keep;
            }
          }
          // P buffer j % 2 is free: its last reader P.V(j-2) was issued before
          // S(j) by the same thread, so the arrival of S(j) means it has landed.
          // A warp whose rows are all zero and whose rows of the buffer already
          // hold zeros leaves them as they are.
          const bool all_zero = zero_half[0] && zero_half[1] && nvalid == TILE;
          if (!(all_zero && ((j & 1) ? zbuf1 : zbuf0))) {
            uint8_t* prow = sm + Smem::P + (2 * X + (j & 1)) * 16384;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(prow + sw128_off(row, c)) =
                  make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
            fence_async_smem();
          }
          // rows whose max moved: acc *= alpha after P.V(j-1) has landed (it
          // was issued a whole tile ago) and before P.V(j) adds to it.  The
          // product is taken in fp32 and rounded to an integer by adding
          // 1.5 * 2^23, whose last mantissa bit is worth 1.  |acc| <= 112 l
          // plus the rounding of earlier rescales, so while l < 2^15 both acc
          // and the product lie below 2^22 and the result is the nearest
          // integer to acc * alpha.  Rows with 2^15 <= l < 2^21 round
          // acc * alpha / 64 (|acc| < 2^28) and scale it back: at most 64 units
          // off, under 1e-4 s_V in O as l >= 2^15 there; rows with l >= 2^21
          // do the same with / 4096 (the host admits N <= 2^19, so
          // 112 l <= 1680 N keeps MB + acc inside int32), at most 4096 units
          // off against l >= 2^21.  The accumulator is kept as MB + acc (MB =
          // the bits of 1.5 * 2^23, written before the first P.V): a short-path
          // row reads MB + acc as the float 1.5 * 2^23 + acc and rescales it
          // with one FMA (within one unit); the other rows subtract MB first.
          // A warp with no large row takes the short loop.
          if (__any_sync(0xffffffffu, moved)) {
            if (!(ok = wait_all(B_PV_DONE + 2 * X + ((j - 1) & 1), ((j - 1) >> 1) & 1, 0x4104))) break;
            tc_fence_after();
            const bool big = l >= 32768.0f, huge = l >= 2097152.0f;
            const bool any_big = __any_sync(0xffffffffu, moved && big);
            uint32_t acc[128];
            tmem_ld128(tO, acc);
            tmem_wait_ld();
            if (moved) {
              if (!any_big) {
                // acc = MB + a with |a| < 2^22: read as a float that is
                // 1.5 * 2^23 + a, and fma(f, alpha, 1.5 * 2^23 (1 - alpha)) rounded
                // to an integer is 1.5 * 2^23 + a alpha within one unit
                const float beta = fmaf(-MAGIC, alpha, MAGIC);
#pragma unroll
                for (int e = 0; e < 128; e += 2) {
                  float r0, r1;
                  fma2(r0, r1, __uint_as_float(acc[e]), __uint_as_float(acc[e + 1]), alpha, alpha, beta, beta);
                  acc[e] = __float_as_uint(r0);
                  acc[e + 1] = __float_as_uint(r1);
                }
              } else {
                const float sc = huge ? alpha * 0.000244140625f : (big ? alpha * 0.015625f : alpha);
                const uint32_t mult = huge ? 4096u : (big ? 64u : 1u),
                               add = (uint32_t)MAGIC_BITS - (uint32_t)MAGIC_BITS * mult;
#pragma unroll
                for (int e = 0; e < 128; e += 2) {
                  float r0, r1;
                  fma2(r0, r1, __int2float_rn((int)(acc[e] - (uint32_t)MAGIC_BITS)),
                       __int2float_rn((int)(acc[e + 1] - (uint32_t)MAGIC_BITS)), sc, sc, MAGIC, MAGIC);
                  acc[e] = __float_as_uint(r0) * mult + add;
                  acc[e + 1] = __float_as_uint(r1) * mult + add;
                }
              }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_st32(tO + 32 * c, acc + 32 * c);
            tmem_wait_st();
          }
          if (j & 1) zbuf1 = all_zero; else zbuf0 = all_zero;
          l = fmaf(l, alpha, (float)L);
          if (dbg_tile && j == a.dbg_kv) {
#pragma unroll
            for (int n = 0; n < 128; ++n) {
              const int w = (int)((pw[2 * (n >> 3) + (n & 1)] >> (8 * ((n & 7) >> 1))) & 0xFF);
              a.dbg_p[row * TILE + n] = n < nvalid ? (int8_t)(w - zp) : (int8_t)-128;
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_P_FULL + 2 * X + (j & 1)]);
        }
        // the last P.V has landed
        if (ok) ok = wait_all(B_PV_DONE + 2 * X + ((nt - 1) & 1), ((nt - 1) >> 1) & 1, 0x4105);
        if (ok) {
          // epilogue: O = acc * s_V / (16 l) -> fp16; loads are warp-collective,
          // stores only for rows < N
          tc_fence_after();
          const float inv = 1.0f / (16.0f * l);
          const float* svb = a.sv + (size_t)bh * D;
          const bool store = grow < P.N && !dbg_run && in_bounds(grow < P.N_pad, err, 0x4013);
          __half* orow = a.o + ((size_t)bh * P.N + (store ? grow : 0)) * D;
          if (P.v_rot) {
            // V was quantised as V H / sqrt(128): the row O' = O H / sqrt(128)
            // goes back through the same (symmetric, orthogonal) transform
            uint32_t acc[128];
            float x[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tO + 32 * c, acc + 32 * c);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 128; ++e) x[e] = (float)(int)(acc[e] - (uint32_t)MAGIC_BITS) * __ldg(svb + e) * inv;
#pragma unroll
            for (int h = 1; h < 128; h <<= 1)
#pragma unroll
              for (int e = 0; e < 128; ++e)
                if (!(e & h)) {
                  const float u = x[e], w = x[e + h];
                  x[e] = u + w;
                  x[e + h] = u - w;
                }
            if (store) {
#pragma unroll
              for (int q = 0; q < 16; ++q) {
                uint32_t hv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const __half2 h2 = __floats2half2_rn(x[8 * q + 2 * e] * 0.08838834764831844055f,
                                                       x[8 * q + 2 * e + 1] * 0.08838834764831844055f);
                  hv[e] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                reinterpret_cast<uint4*>(orow)[q] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
              }
            }
          } else {
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t acc[16];
            tmem_ld16(tO + 16 * c, acc);
            tmem_wait_ld();
            uint32_t hv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float x0 = (float)(int)(acc[2 * e] - (uint32_t)MAGIC_BITS) * __ldg(svb + 16 * c + 2 * e) * inv;
              const float x1 =
                  (float)(int)(acc[2 * e + 1] - (uint32_t)MAGIC_BITS) * __ldg(svb + 16 * c + 2 * e + 1) * inv;
              const __half2 h2 = __floats2half2_rn(x0, x1);
              hv[e] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            if (store) {
              uint4* dst = reinterpret_cast<uint4*>(orow + 16 * c);
              dst[0] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
              dst[1] = make_uint4(hv[4], hv[5], hv[6], hv[7]);
            }
          }
          }
        }
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ bulk-copy producer
    // The INT8 operand images are laid out as the MMA reads them (128-byte
    // swizzled, K-major), so every tile is one contiguous 16 KB copy.
    if (lane == 0) {
      const uint8_t* qsrc = a.qimg + ((size_t)bh * nt + qt0) * 16384;
      const bool q_ok = in_bounds(qt0 + (hasB ? 2 : 1) <= nt, err, 0x4014);
      if (!q_ok) *abort_flag = 1;   // every wait gives up; nothing is copied
      if (q_ok) {
        mbar_expect_tx(&bar[B_QFULL], hasB ? 32768u : 16384u);
        bulk_g2s(sm + Smem::QA, qsrc, 16384, &bar[B_QFULL]);
        if (hasB) bulk_g2s(sm + Smem::QB, qsrc + 16384, 16384, &bar[B_QFULL]);
      }
      const uint8_t* kb = a.kimg + (size_t)bh * nt * 16384;
      const uint8_t* vb = a.vimg + (size_t)bh * nt * 16384;
      int issued = 0;
      for (int j = 0; q_ok && j < nt; ++j) {
        const int st = j % OP_STAGES;
        if (j >= OP_STAGES && !mbar_wait_abortable(&bar[B_OP_EMPTY + st], ((j / OP_STAGES) - 1) & 1, abort_flag,
                                                   limit, err, 0x4201))
          break;
        uint8_t* dst = sm + Smem::OP + st * 32768;
        if (!in_bounds(j < nt && st < OP_STAGES, err, 0x4015)) {
          *abort_flag = 1;
          break;
        }
        mbar_expect_tx(&bar[B_OP_FULL + st], 32768u);
        bulk_g2s(dst, kb + (size_t)j * 16384, 16384, &bar[B_OP_FULL + st]);
        bulk_g2s(dst + 16384, vb + (size_t)j * 16384, 16384, &bar[B_OP_FULL + st]);
        issued = j + 1;
      }
      if (*abort_flag) {   // let every copy still in flight land before the CTA exits
        if (q_ok) mbar_wait(&bar[B_QFULL], 0, limit, err, 0x4203);
        for (int j = issued > OP_STAGES ? issued - OP_STAGES : 0; j < issued; ++j)
          mbar_wait(&bar[B_OP_FULL + j % OP_STAGES], (j / OP_STAGES) & 1, limit, err, 0x4204);
      }
    }
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------ MMA issuers
    // One thread per query tile, each blocked on its own tile's barriers.
    // Tile X computes S_X(j+1) = Q_X K(j+1)^T as soon as its softmax warps
    // have S_X(j) in registers, so the next S is ready when they finish tile
    // j; O_X += W_X(j) V(j) follows once W_X(j) is stored (and O_X rescaled).
    // MMAs of one thread complete in issue order; the two threads' MMAs touch
    // disjoint TMEM and only read the shared operand stages, whose release
    // counts one commit from each thread.
    const int X = warp - 9;
    if (lane == 0 && (X == 0 || hasB)) {
      const uint32_t qa = smem_u32(sm + (X ? Smem::QB : Smem::QA));
      const uint32_t pbase = smem_u32(sm + Smem::P + 2 * X * 16384);
      const uint32_t op = smem_u32(sm + Smem::OP);
      const uint32_t tS = tbase + X * 128, tO = tbase + 256 + X * 128;
      auto wait = [&](int b, uint32_t parity, uint32_t site) {
        return mbar_spin_abortable(&bar[b], parity, abort_flag, limit, err, site);
      };
      // A 32-byte step along K adds 2 to a descriptor's address field
      // (address / 16 in bits 0-13; every operand lies below 2^18 bytes and
      // starts on a 1024-byte boundary, so the field never carries).
      const uint64_t dq = sw128_desc(qa);
      auto issue_S = [&](int j) {   // S_X(j) = 256 Q_X K(j)^T
        const uint64_t dk = sw128_desc(op + (j % OP_STAGES) * 32768);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_i8(tS, dq + 2 * kk, dk + 2 * kk, IDESC_QK, kk > 0);
        umma_commit(&bar[B_S_FULL + X]);
      };
      bool ok = wait(B_QFULL, 0, 0x4301) && wait(B_OP_FULL, 0, 0x4302);
      if (ok) {
        tc_fence_after();
        issue_S(0);
      }
      for (int j = 0; ok && j < nt; ++j) {
        if (j + 1 < nt) {
          if (!(ok = wait(B_S_EMPTY + X, j & 1, 0x4303))) break;
          if (!(ok = wait(B_OP_FULL + (j + 1) % OP_STAGES, ((j + 1) / OP_STAGES) & 1, 0x4304))) break;
          tc_fence_after();
          issue_S(j + 1);
        }
        if (!(ok = wait(B_P_FULL + 2 * X + (j & 1), (j >> 1) & 1, 0x4305))) break;
        tc_fence_after();
        const uint64_t dv = sw128_desc(op + (j % OP_STAGES) * 32768 + 16384);   // O_X += W_X(j) V(j)
        const uint64_t dp = sw128_desc(pbase + (j & 1) * 16384);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_i8(tO, dp + 2 * kk, dv + 2 * kk, IDESC_PV, 1);   // onto MB
        umma_commit(&bar[B_PV_DONE + 2 * X + (j & 1)]);
        umma_commit(&bar[B_OP_EMPTY + j % OP_STAGES]);
      }
      // every MMA this thread issued completes before TMEM is released
      umma_commit(&bar[B_DRAIN + X]);
      mbar_wait(&bar[B_DRAIN + X], 0, limit, err, 0x4308);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace

cudaError_t launch_int4_attention(const Prob& p, const uint8_t* q4, const uint8_t* k4, const uint8_t* v4t,
                                  const float* sq, const float* sk, const float* sv, __half* o, void* ws, int dbg_bh,
                                  int dbg_qtile, int dbg_kv, int32_t* dbg_s, int8_t* dbg_p, cudaStream_t st) {
  const int smem = Smem::BYTES + 1024;   // > half the SM: one CTA per SM owns all 512 TMEM columns
  auto kernel = dbg_s ? int4_attn_kernel<true> : int4_attn_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // The setmaxnreg split assumes the kernel launches with LAUNCH_REGS per
  // thread; with fewer, the softmax warpgroups' increase could never be
  // granted.  Refuse to launch rather than risk that.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != LAUNCH_REGS) return cudaErrorInvalidConfiguration;
  const WsLayout L = ws_layout(p);
  uint8_t* img = static_cast<uint8_t*>(ws) + L.img;
  const size_t plane = (size_t)p.BH * p.N_pad * D;   // bytes of one operand image set
  const size_t units = plane / 32;                   // 16 packed bytes -> 32 image bytes
  expand_kernel<<<dim3((unsigned)((units + 255) / 256), 3), 256, 0, st>>>(q4, k4, v4t, img, img + plane,
                                                                          img + 2 * plane, units,
                                                                          &static_cast<WsHeader*>(ws)->err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  KernelArgs a{p, img, img + plane, img + 2 * plane, sq, sk, sv, o, static_cast<WsHeader*>(ws), wait_limit(),
               dbg_bh, dbg_qtile, dbg_kv,
               dbg_s, dbg_p};
  const int n_qt = p.N_pad / TILE;
  const dim3 grid = dbg_s ? dim3(1, 1) : dim3((n_qt + 1) / 2, p.BH);
  kernel<<<grid, NUM_THREADS, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace ra
