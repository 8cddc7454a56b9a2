// ra_api.cu -- host side of the C ABI declared in include/rotate_attn.h:
// argument validation, RoPE/rotation coefficient tables, workspace layout,
// error reporting and kernel launches.  No allocation anywhere: every buffer
// is the caller's.
#include <atomic>
#include <cstdarg>
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <vector>

#include <cuda_runtime.h>

#include "ra_internal.h"

namespace {

thread_local char g_detail[256] = "";
std::atomic<uint32_t> g_wait_limit_us{0};
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;   // 2 s of wall-clock time per wait

ra_status fail(ra_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
ra_status fail(ra_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return s;
}

ra_status cuda_fail(cudaError_t e, const char* what) {
  cudaGetLastError();   // clear the sticky-free error so later calls start clean
  return fail(RA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

uint64_t fnv1a(const void* data, size_t n, uint64_t h = 1469598103934665603ull) {
  const unsigned char* b = static_cast<const unsigned char*>(data);
  for (size_t i = 0; i < n; ++i) h = (h ^ b[i]) * 1099511628211ull;
  return h;
}

// Validates and derives the kernel-side sizes.
ra_status derive(const ra_problem* p, ra::Prob* out) {
  if (p == nullptr) return fail(RA_ERR_INVALID_ARG, "problem is NULL");
  if (p->B < 1 || p->H < 1) return fail(RA_ERR_INVALID_ARG, "B and H must be >= 1 (got %d, %d)", p->B, p->H);
  if (p->d != ra::D) return fail(RA_ERR_UNSUPPORTED, "head_dim %d: only 128 is built", p->d);
  if (p->F < 0 || p->Hh < 0 || p->W < 0 || p->n_text < 0)
    return fail(RA_ERR_INVALID_ARG, "negative grid or text size");
  const long long nv = (long long)p->F * p->Hh * p->W;
  const long long N = nv + p->n_text;
  if (N < 1) return fail(RA_ERR_INVALID_ARG, "empty sequence (N = 0)");
  const bool any_zero = p->F == 0 || p->Hh == 0 || p->W == 0;
  const bool all_zero = p->F == 0 && p->Hh == 0 && p->W == 0;
  if (any_zero && !all_zero) return fail(RA_ERR_INVALID_ARG, "video grid with a zero axis (use 0x0x0 for text only)");
  int sum = 0;
  for (int s = 0; s < 3; ++s) {
    if (p->split[s] <= 0 || (p->split[s] & 1))
      return fail(RA_ERR_INVALID_ARG, "RoPE segment %d size %d must be even and positive", s, p->split[s]);
    sum += p->split[s];
  }
  if (sum != p->d) return fail(RA_ERR_INVALID_ARG, "RoPE split sums to %d, head_dim is %d", sum, p->d);
  if (p->rot < RA_ROT_NONE || p->rot > RA_ROT_BLOCKS_HALF)
    return fail(RA_ERR_INVALID_ARG, "rotation mode %d unknown", p->rot);
  const bool blocks = p->rot == RA_ROT_BLOCKS_INTERLEAVED || p->rot == RA_ROT_BLOCKS_HALF;
  if (blocks) {
    if (p->blocks == nullptr) return fail(RA_ERR_INVALID_ARG, "rotation mode %d needs the pair blocks", p->rot);
    for (int q = 0; q < p->d / 2; ++q) {
      const double* r = p->blocks + 4 * q;
      const double e0 = r[0] * r[0] + r[1] * r[1] - 1.0, e1 = r[2] * r[2] + r[3] * r[3] - 1.0;
      const double e2 = r[0] * r[2] + r[1] * r[3];
      if (!(std::fabs(e0) < 1e-6 && std::fabs(e1) < 1e-6 && std::fabs(e2) < 1e-6))
        return fail(RA_ERR_INVALID_ARG, "pair block %d is not orthogonal", q);
    }
  }
  if (!(p->theta > 0.0) || !std::isfinite(p->theta)) return fail(RA_ERR_INVALID_ARG, "RoPE base must be > 0");
  if (p->p_mode != RA_P_RANGE_OPTIMIZED && p->p_mode != RA_P_SYMMETRIC)
    return fail(RA_ERR_INVALID_ARG, "P quantisation mode %d unknown", p->p_mode);
  if (p->v_rot != 0 && p->v_rot != 1) return fail(RA_ERR_INVALID_ARG, "v_rot must be 0 or 1, not %d", p->v_rot);
  const long long Np = (N + ra::TILE - 1) / ra::TILE * ra::TILE;
  // The INT4 attention's int32 P.V accumulator holds the offset 0x4B400000
  // plus up to 112 x (sum of P weights) <= 112 x 15 N: 2^19 tokens keep it
  // inside the int32 range.
  if (N > ra::MAX_TOKENS)
    return fail(RA_ERR_UNSUPPORTED, "sequence too long: %lld tokens (at most %d)", N, ra::MAX_TOKENS);
  if ((long long)p->B * p->H > 65535) return fail(RA_ERR_UNSUPPORTED, "B*H > 65535");
  if (out) {
    ra::Prob& P = *out;
    P.B = p->B;
    P.H = p->H;
    P.BH = p->B * p->H;
    P.N = (int)N;
    P.N_pad = (int)Np;
    P.n_video = (int)nv;
    P.F = p->F;
    P.Hh = p->Hh;
    P.W = p->W;
    P.rot = p->rot;
    P.p_mode = p->p_mode;
    P.v_rot = p->v_rot;
    const int npos[3] = {p->F > 0 ? p->F : 1, p->Hh > 0 ? p->Hh : 1, p->W > 0 ? p->W : 1};
    int off = 0, toff = 0;
    for (int s = 0; s < 3; ++s) {
      P.split[s] = p->split[s];
      P.off[s] = off;
      off += p->split[s];
      P.npos[s] = npos[s];
      P.tab_off[s] = toff;
      P.tab_q[s] = (p->split[s] / 2 + 3) / 4;
      toff += npos[s] * 4 * P.tab_q[s];
    }
    P.fastdiv = 1;
    const uint64_t divs[2] = {(uint64_t)(p->W > 0 ? p->W : 1), (uint64_t)(p->W > 0 ? p->W : 1) * (p->Hh > 0 ? p->Hh : 1)};
    uint32_t mags[2];
    for (int i = 0; i < 2; ++i) {
      const uint64_t d = divs[i];
      const uint64_t m = ((1ull << 32) + d - 1) / d;   // ceil(2^32 / d)
      mags[i] = m >> 32 ? 0u : (uint32_t)m;            // d = 1: identity
      if (d > 1 && (uint64_t)nv * (m * d - (1ull << 32)) >= (1ull << 32)) P.fastdiv = 0;
    }
    P.m_w = mags[0];
    P.m_hw = mags[1];
    P.n_tab = toff;
    P.n_tab_all = toff + p->d / 2;
    P.half4 = 1;
    for (int s = 0; s < 3; ++s)
      if ((P.off[s] & 3) || ((p->split[s] / 2) & 3)) P.half4 = 0;
    // what the tables depend on; B and H only size the buffers (checked on the
    // host), so one prepared workspace serves any batch and head count it fits
    uint64_t h = fnv1a(&p->d, sizeof(int) * 5);
    h = fnv1a(p->split, sizeof(p->split), h);
    h = fnv1a(&p->theta, sizeof(double), h);
    h = fnv1a(&p->rot, sizeof(int), h);
    if (blocks) h = fnv1a(p->blocks, sizeof(double) * 4 * (size_t)(p->d / 2), h);
    P.signature = h | 1ull;   // never 0, so a zeroed workspace never matches
  }
  return RA_OK;
}

// Coefficients {cos a, sin a, (cos a + sin a)/sqrt2, (cos a - sin a)/sqrt2}
// per (segment, position, pair), a = pos * theta^(-2j/d_s), each computed in
// float64 and rounded once to fp32.  A position's block of segment s has
// 4 q slots (q = ceil(d_s / 8)), pair j at slot (j % 4) q + j / 4, the rest
// zero: the 16 threads of a row hold pairs 4g .. 4g + 3 (channels 8g .. 8g +
// 7), so for each of their four pairs they read consecutive slots.
void build_tables(const ra_problem* p, const ra::Prob& P, float* out) {
  const bool blocks_mode = p->rot == RA_ROT_BLOCKS_INTERLEAVED || p->rot == RA_ROT_BLOCKS_HALF;
  std::fill(out, out + 4 * (size_t)P.n_tab, 0.0f);   // the unused slots of each block
  for (int s = 0; s < 3; ++s) {
    const int half = p->split[s] / 2;
    for (int pos = 0; pos < P.npos[s]; ++pos)
      for (int j = 0; j < half; ++j) {
        const double w = std::pow(p->theta, -(double)(2 * j) / (double)p->split[s]);
        const double a = (double)pos * w;
        const double ca = std::cos(a), sa = std::sin(a);
        const int q = P.tab_q[s];
        float* e = out + 4 * ((size_t)P.tab_off[s] + (size_t)pos * 4 * q + (size_t)(j % 4) * q + j / 4);
        if (p->rot == RA_ROT_BLOCKS_INTERLEAVED) {   // R times the RoPE rotation, per (pos, pair)
          const double* r = p->blocks + 4 * (P.off[s] / 2 + j);
          e[0] = (float)(r[0] * ca + r[1] * sa);
          e[1] = (float)(r[1] * ca - r[0] * sa);
          e[2] = (float)(r[2] * ca + r[3] * sa);
          e[3] = (float)(r[3] * ca - r[2] * sa);
        } else {
          e[0] = (float)ca;
          e[1] = (float)sa;
          e[2] = (float)((ca + sa) * M_SQRT1_2);
          e[3] = (float)((ca - sa) * M_SQRT1_2);
        }
      }
  }
  // pair blocks, rounded to fp32 (used by BLOCKS_HALF), zero otherwise
  for (int q = 0; q < p->d / 2; ++q)
    for (int k = 0; k < 4; ++k) out[4 * ((size_t)P.n_tab + q) + k] = blocks_mode ? (float)p->blocks[4 * q + k] : 0.0f;
}

struct QkvLayout {
  size_t q4, k4, v4t, sq, sk, sv, vsum, total;
};

QkvLayout qkv_layout(const ra::Prob& P) {
  QkvLayout L;
  size_t o = 0;
  const size_t packed = (size_t)P.BH * P.N_pad * (ra::D / 2);
  L.q4 = o;
  o = ra::align256(o + packed);
  L.k4 = o;
  o = ra::align256(o + packed);
  L.v4t = o;
  o = ra::align256(o + packed);
  L.sq = o;
  o = ra::align256(o + sizeof(float) * (size_t)P.BH * (P.N_pad / ra::QK_BLOCK));
  L.sk = o;
  o = ra::align256(o + sizeof(float) * (size_t)P.BH * (P.N_pad / ra::QK_BLOCK));
  L.sv = o;
  o = ra::align256(o + sizeof(float) * (size_t)P.BH * ra::D);
  L.vsum = o;
  o = ra::align256(o + sizeof(int32_t) * (size_t)P.BH * (P.N_pad / ra::QK_BLOCK) * ra::D);
  L.total = o;
  return L;
}

enum class WsUse { prologue, int4, fp16 };

ra_status check_ws(const ra::Prob& P, const void* ws, size_t bytes, WsUse use) {
  if (!aligned16(ws)) return fail(RA_ERR_INVALID_ARG, "workspace pointer NULL or not 16-byte aligned");
  const ra::WsLayout L = ra::ws_layout(P);
  const size_t need = use == WsUse::fp16 ? L.total_fp16 : (use == WsUse::int4 ? L.base_bytes : L.pro_bytes);
  if (bytes < need) return fail(RA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", bytes, need);
  return RA_OK;
}

ra_status check_qkv4(const ra_qkv4* t) {
  if (t == nullptr) return fail(RA_ERR_INVALID_ARG, "ra_qkv4 is NULL");
  if (!aligned16(t->q4) || !aligned16(t->k4) || !aligned16(t->v4t) || !aligned16(t->sq) || !aligned16(t->sk) ||
      !aligned16(t->sv) || !aligned16(t->vsum))
    return fail(RA_ERR_INVALID_ARG, "an ra_qkv4 pointer is NULL or not 16-byte aligned");
  return RA_OK;
}

}  // namespace

namespace ra {
uint64_t wait_limit() {
  const uint32_t us = g_wait_limit_us.load(std::memory_order_relaxed);
  return us ? 1000ull * us : kDefaultWaitLimitNs;
}
ra_status derive_problem(const ra_problem* p, Prob* out) { return derive(p, out); }
void build_coef_tables(const ra_problem* p, const Prob& P, float* out) { build_tables(p, P, out); }
void set_error_detail(const char* msg) { snprintf(g_detail, sizeof(g_detail), "%s", msg); }
}  // namespace ra

extern "C" {

int ra_seq_len(const ra_problem* p) {
  ra::Prob P;
  return derive(p, &P) == RA_OK ? P.N : -1;
}

int ra_seq_pad(const ra_problem* p) {
  ra::Prob P;
  return derive(p, &P) == RA_OK ? P.N_pad : -1;
}

ra_status ra_validate(const ra_problem* p) { return derive(p, nullptr); }

size_t ra_qkv4_bytes(const ra_problem* p) {
  ra::Prob P;
  if (derive(p, &P) != RA_OK) return 0;
  return qkv_layout(P).total;
}

ra_status ra_qkv4_bind(const ra_problem* p, void* base, size_t bytes, ra_qkv4* out) {
  ra::Prob P;
  ra_status st = derive(p, &P);
  if (st != RA_OK) return st;
  if (out == nullptr) return fail(RA_ERR_INVALID_ARG, "output ra_qkv4 is NULL");
  if (base == nullptr || (reinterpret_cast<uintptr_t>(base) & 255u))
    return fail(RA_ERR_INVALID_ARG, "qkv4 buffer NULL or not 256-byte aligned");
  const QkvLayout L = qkv_layout(P);
  if (bytes < L.total) return fail(RA_ERR_INVALID_ARG, "qkv4 buffer has %zu bytes, needs %zu", bytes, L.total);
  char* b = static_cast<char*>(base);
  out->q4 = reinterpret_cast<uint8_t*>(b + L.q4);
  out->k4 = reinterpret_cast<uint8_t*>(b + L.k4);
  out->v4t = reinterpret_cast<uint8_t*>(b + L.v4t);
  out->sq = reinterpret_cast<float*>(b + L.sq);
  out->sk = reinterpret_cast<float*>(b + L.sk);
  out->sv = reinterpret_cast<float*>(b + L.sv);
  out->vsum = reinterpret_cast<int32_t*>(b + L.vsum);
  return RA_OK;
}

size_t ra_workspace_bytes(const ra_problem* p, int with_fp16_path) {
  ra::Prob P;
  if (derive(p, &P) != RA_OK) return 0;
  const ra::WsLayout L = ra::ws_layout(P);
  return with_fp16_path ? L.total_fp16 : L.base_bytes;
}

size_t ra_tables_floats(const ra_problem* p) {
  ra::Prob P;
  if (derive(p, &P) != RA_OK) return 0;
  return 4 * (size_t)P.n_tab_all;
}

ra_status ra_build_tables_host(const ra_problem* p, float* out, size_t n_floats) {
  ra::Prob P;
  ra_status st = derive(p, &P);
  if (st != RA_OK) return st;
  if (out == nullptr || n_floats < 4 * (size_t)P.n_tab_all)
    return fail(RA_ERR_INVALID_ARG, "table buffer NULL or smaller than %zu floats", 4 * (size_t)P.n_tab_all);
  build_tables(p, P, out);
  return RA_OK;
}

ra_status ra_prepare(const ra_problem* p, void* ws, size_t ws_bytes, ra_stream stream) {
  ra::Prob P;
  ra_status st = derive(p, &P);
  if (st != RA_OK) return st;
  if ((st = check_ws(P, ws, ws_bytes, WsUse::prologue)) != RA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ra::WsLayout L = ra::ws_layout(P);
  std::vector<float> tab(4 * (size_t)P.n_tab_all);
  build_tables(p, P, tab.data());
  ra::WsHeader hdr{};
  hdr.signature = P.signature;
  char* base = static_cast<char*>(ws);
  // Pageable source: the runtime stages both copies before returning.
  cudaError_t e = cudaMemcpyAsync(base + L.tables, tab.data(), sizeof(float) * tab.size(), cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "table upload");
  e = cudaMemcpyAsync(base, &hdr, sizeof(hdr), cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "header upload");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "prepare");
  return RA_OK;
}

ra_status ra_rotate_quantize_qkv(const ra_problem* p, const void* q, const void* k, const void* v,
                                 const ra_qkv4* out, void* ws, size_t ws_bytes, ra_stream stream) {
  ra::Prob P;
  ra_status st = derive(p, &P);
  if (st != RA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v))
    return fail(RA_ERR_INVALID_ARG, "q, k or v NULL or not 16-byte aligned");
  if ((st = check_qkv4(out)) != RA_OK) return st;
  if ((st = check_ws(P, ws, ws_bytes, WsUse::prologue)) != RA_OK) return st;
  cudaError_t e = ra::launch_prologue(P, static_cast<const __half*>(q), static_cast<const __half*>(k),
                                      static_cast<const __half*>(v), out->q4, out->k4, out->v4t, out->sq, out->sk,
                                      out->sv, out->vsum, ws, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "prologue launch");
}

ra_status ra_int4_attention_fwd(const ra_problem* p, const ra_qkv4* in, void* o, void* ws, size_t ws_bytes,
                                ra_stream stream) {
  ra::Prob P;
  ra_status st = derive(p, &P);
  if (st != RA_OK) return st;
  if ((st = check_qkv4(in)) != RA_OK) return st;
  if (!aligned16(o)) return fail(RA_ERR_INVALID_ARG, "output NULL or not 16-byte aligned");
  if ((st = check_ws(P, ws, ws_bytes, WsUse::int4)) != RA_OK) return st;
  cudaError_t e = ra::launch_int4_attention(P, in->q4, in->k4, in->v4t, in->sq, in->sk, in->sv,
                                            static_cast<__half*>(o), ws, -1, -1, -1, nullptr, nullptr,
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "int4 attention launch");
}

ra_status ra_fp16_attention_fwd(const ra_problem* p, const void* q, const void* k, const void* v, void* o, void* ws,
                                size_t ws_bytes, ra_stream stream) {
  ra::Prob P;
  ra_status st = derive(p, &P);
  if (st != RA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(RA_ERR_INVALID_ARG, "q, k, v or o NULL or not 16-byte aligned");
  if ((st = check_ws(P, ws, ws_bytes, WsUse::fp16)) != RA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = ra::launch_fp16_prologue(P, static_cast<const __half*>(q), static_cast<const __half*>(k),
                                           static_cast<const __half*>(v), ws, s);
  if (e != cudaSuccess) return cuda_fail(e, "fp16 prologue launch");
  e = ra::launch_fp16_attention(P, static_cast<__half*>(o), ws, s);
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "fp16 attention launch");
}

ra_status ra_check_device_error(void* ws, ra_stream stream) {
  if (!aligned16(ws)) return fail(RA_ERR_INVALID_ARG, "workspace pointer NULL or not 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  ra::DeviceErr err{};
  e = cudaMemcpy(&err, ws, sizeof(err), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "error word read");
  if (err.word == 0) return RA_OK;
  e = cudaMemset(ws, 0, sizeof(err));
  if (e != cudaSuccess) return cuda_fail(e, "error word clear");
  if (err.word & ra::DEVERR_WORKSPACE)
    return fail(RA_ERR_WORKSPACE, "workspace not prepared for this problem (site 0x%x)", err.site);
  if (err.word & ra::DEVERR_BOUNDS) return fail(RA_ERR_DEVICE_BOUNDS, "device bounds check (site 0x%x)", err.site);
  return fail(RA_ERR_DEVICE_TIMEOUT, "bounded device wait ran out (site 0x%x)", err.site);
}

const char* ra_status_string(ra_status s) {
  switch (s) {
    case RA_OK: return "ok";
    case RA_ERR_INVALID_ARG: return "invalid argument";
    case RA_ERR_UNSUPPORTED: return "unsupported";
    case RA_ERR_WORKSPACE: return "workspace too small or not prepared";
    case RA_ERR_CUDA: return "CUDA error";
    case RA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case RA_ERR_DEVICE_BOUNDS: return "device bounds check failed";
  }
  return "unknown status";
}

const char* ra_last_error_detail(void) { return g_detail; }

ra_status ra_debug_int4_tile(const ra_problem* p, const ra_qkv4* in, int bh, int q_tile, int kv_tile,
                             int32_t* s_out, int8_t* p_out, void* ws, size_t ws_bytes, ra_stream stream) {
  ra::Prob P;
  ra_status st = derive(p, &P);
  if (st != RA_OK) return st;
  if ((st = check_qkv4(in)) != RA_OK) return st;
  if ((st = check_ws(P, ws, ws_bytes, WsUse::int4)) != RA_OK) return st;
  if (bh < 0 || bh >= P.BH || q_tile < 0 || q_tile >= P.N_pad / ra::TILE || kv_tile < 0 ||
      kv_tile >= P.N_pad / ra::TILE)
    return fail(RA_ERR_INVALID_ARG, "debug tile index out of range");
  if (!aligned16(s_out) || !aligned16(p_out)) return fail(RA_ERR_INVALID_ARG, "debug outputs NULL or misaligned");
  cudaError_t e = ra::launch_int4_attention(P, in->q4, in->k4, in->v4t, in->sq, in->sk, in->sv, nullptr, ws, bh,
                                            q_tile, kv_tile, s_out, p_out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "debug launch");
}

void ra_debug_set_wait_timeout_us(uint32_t microseconds) {
  g_wait_limit_us.store(microseconds, std::memory_order_relaxed);
}

ra_status ra_debug_timeout_probe(void* ws, size_t ws_bytes, ra_stream stream) {
  if (!aligned16(ws) || ws_bytes < sizeof(ra::WsHeader))
    return fail(RA_ERR_INVALID_ARG, "workspace NULL, misaligned or too small");
  cudaError_t e = ra::launch_timeout_probe(ws, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "timeout probe launch");
}

ra_status ra_debug_ex2(const float* x, float* y, int n, ra_stream stream) {
  if (n < 0 || (n > 0 && (!aligned16(x) || !aligned16(y))))
    return fail(RA_ERR_INVALID_ARG, "ex2 probe: n < 0 or x, y NULL or misaligned");
  cudaError_t e = ra::launch_ex2_probe(x, y, n, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "ex2 probe launch");
}

ra_status ra_measure_mma_i8(int n, int iters, int ctas, void* ws, size_t ws_bytes, ra_stream stream) {
  if (n != 128 && n != 256) return fail(RA_ERR_INVALID_ARG, "MMA width %d: 128 or 256", n);
  if (iters < 1 || ctas < 1) return fail(RA_ERR_INVALID_ARG, "iters and ctas must be >= 1");
  if (!aligned16(ws) || ws_bytes < sizeof(ra::WsHeader))
    return fail(RA_ERR_INVALID_ARG, "workspace NULL, misaligned or too small");
  cudaError_t e = ra::launch_mma_i8_rate(n, iters, ctas, ws, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "MMA rate launch");
}

}  // extern "C"
