// ra_internal.h -- derived problem sizes, workspace layout and the launch
// functions shared by the C ABI (ra_api.cu) and the kernel files.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "ra_sm100.cuh"
#include "../../include/rotate_attn.h"

namespace ra {

constexpr int D = 128;          // head_dim
constexpr int QK_BLOCK = 64;    // tokens per Q/K quantisation block
constexpr int TILE = 128;       // query rows per CTA tile and keys per KV tile
constexpr int MAX_TOKENS = RA_MAX_TOKENS;   // longest sequence: 0x4B400000 + 1680 N < 2^31 (P.V accumulator)

// Problem with the sizes the kernels need, computed once on the host.
struct Prob {
  int B, H, BH;
  int N, N_pad, n_video;
  int F, Hh, W;
  int split[3], off[3];         // segment sizes and first channel of each segment
  int npos[3];                  // positions per axis: F, Hh, W
  int tab_off[3];               // first table entry of each segment
  int tab_q[3];                 // ceil(split[s] / 8): a position's block of segment s holds 4 tab_q
                                // entries, pair j at slot (j % 4) tab_q + j / 4
  int n_tab;                    // RoPE table entries (each: cos, sin, alpha, beta, or for
                                // BLOCKS_INTERLEAVED the merged m00, m01, m10, m11)
  int n_tab_all;                // n_tab + d/2 pair-block entries (r00, r01, r10, r11)
  // token -> (f, h, w) without integer division: n / d = umulhi(n, m) for
  // m = ceil(2^32 / d), exact while n * (m d - 2^32) < 2^32 for every video
  // token (checked on the host; fastdiv = 0 falls back to / and %); m = 0
  // stands for d = 1
  uint32_t m_w, m_hw;           // divisors W and Hh * W
  int fastdiv;
  int rot;
  int half4;                    // every segment and half-segment boundary is a multiple of 4
  int p_mode;                   // ra_p_mode
  int v_rot;                    // 1: Hadamard on V, undone on O (INT4 path)
  uint64_t signature;
};

// Workspace layout (all offsets 256-byte aligned).
struct WsHeader {
  DeviceErr err;                // error word + first reporting site
  uint32_t reserved0[2];
  unsigned long long signature; // problem signature written by ra_prepare
};

struct WsLayout {
  size_t tables;                // float4 [n_tab]
  size_t vamax;                 // uint32 [BH][128]: fp32 bits of per-channel amax of V
  size_t pro_bytes;             // end of the part the prologue needs
  size_t img;                   // INT4 attention: INT8 operand images of Q, K, V^T,
                                // 3 x [BH][N_pad / 128][16 KB]
  size_t base_bytes;            // end of the part the INT4 path needs
  size_t qr, kr, vt;            // FP16 path: operand images of RoPE-encoded Q, K and of V^T,
                                // [BH][N_pad / 128][32 KB] each (two swizzled 16 KB atoms)
  size_t total_fp16;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(const Prob& p) {
  WsLayout L;
  size_t o = align256(sizeof(WsHeader));
  L.tables = o;
  o = align256(o + sizeof(float) * 4 * (size_t)p.n_tab_all);
  L.vamax = o;
  o = align256(o + sizeof(uint32_t) * (size_t)p.BH * D);
  L.pro_bytes = o;
  L.img = o;
  o = align256(o + 3 * (size_t)p.BH * p.N_pad * D);
  L.base_bytes = o;
  size_t plane = (size_t)p.BH * p.N_pad * D * 2;
  L.qr = o;
  o = align256(o + plane);
  L.kr = o;
  o = align256(o + plane);
  L.vt = o;
  o = align256(o + plane);
  L.total_fp16 = o;
  return L;
}

// Launches (stream-ordered; return the launch status).
cudaError_t launch_prologue(const Prob& p, const __half* q, const __half* k, const __half* v, uint8_t* q4,
                            uint8_t* k4, uint8_t* v4t, float* sq, float* sk, float* sv, int32_t* vsum,
                            void* ws, cudaStream_t st);
cudaError_t launch_fp16_prologue(const Prob& p, const __half* q, const __half* k, const __half* v, void* ws,
                                 cudaStream_t st);
cudaError_t launch_int4_attention(const Prob& p, const uint8_t* q4, const uint8_t* k4, const uint8_t* v4t,
                                  const float* sq, const float* sk, const float* sv, __half* o, void* ws,
                                  int dbg_bh, int dbg_qtile, int dbg_kv, int32_t* dbg_s, int8_t* dbg_p,
                                  cudaStream_t st);
cudaError_t launch_fp16_attention(const Prob& p, __half* o, void* ws, cudaStream_t st);
cudaError_t launch_timeout_probe(void* ws, cudaStream_t st);
cudaError_t launch_mma_i8_rate(int n, int iters, int ctas, void* ws, cudaStream_t st);
cudaError_t launch_ex2_probe(const float* x, float* y, int n, cudaStream_t st);

// Wall-clock limit (ns) of every bounded device-side wait.
uint64_t wait_limit();

// Host helpers shared with the allocation-free entry point (ra_noalloc.cu):
// problem validation with derived sizes, and the coefficient table builder.
ra_status derive_problem(const ra_problem* p, Prob* out);
void build_coef_tables(const ra_problem* p, const Prob& P, float* out);
void set_error_detail(const char* msg);

}  // namespace ra
