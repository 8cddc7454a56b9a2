// ra_host.cu -- the INT4 forward from and to host memory, with the copies
// overlapped with the kernels.
//
// Heads are independent in every step of the path (Q/K blocks, V channel
// scales and the attention all live inside one (b, h)), so the flattened
// B*H heads are cut into chunks of consecutive heads, each a problem of its
// own with B = 1.  Four streams form a pipeline over the chunks:
//
//   copy-in stream   : q, k, v of chunk c, host -> slot c % 3
//   compute lane c%2 : prologue + INT4 attention of chunk c (slot c % 3);
//                      lane 0 is the caller's stream, lane 1 one of ours
//   copy-out stream  : o of chunk c, slot c % 3 -> host
//
// so that the host->device copy of chunk c+1 and the device->host copy of
// chunk c-1 run on the copy engines while chunk c is computed, and the
// kernels of chunk c+1 fill the SMs that the last wave of chunk c leaves idle
// (each slot has its own quantised tensors and workspace).  Events order the
// reuse of the three slots: the copy-in of chunk c may start once chunk c - 3
// has been computed, so it runs up to two chunks ahead of the kernels.  The
// call blocks until o is written.
#include <algorithm>
#include <cstdio>
#include <vector>

#include <cuda_runtime.h>

#include "ra_internal.h"

namespace {

constexpr int kDefaultChunks = 8;   // chunks of the largest size when the caller passes 0
constexpr int kSlots = 3;           // staging slots: chunk c uses slot c % kSlots

struct HostPlan {
  std::vector<int> heads;     // heads of every chunk, in order
  int BH, per;                // flattened heads; the largest chunk
  ra_problem chunk;           // B = 1, H = per (sizes the regions below)
  size_t head_bytes;          // one head of one fp16 tensor: N * 128 * 2
  size_t ws, qkv4, io;        // per-slot region sizes (256-aligned)
  size_t slot, total;         // one slot: workspace, quantised tensors, q, k, v, o
};

// Chunk sizes.  Given heads_per_chunk > 0: equal chunks (the last one takes
// the remainder).  Given 0: chunks of about B*H/8 heads, entered by the ramp
// 1, 1, 2, 2, 3, 3, 4, 4, ... and left by ..., 3, 2, 1, so that the first
// kernels wait only for a one-head copy and the last copy-out is of one
// head.  A head's copy-in takes about 0.85 of its compute; with three slots
// the copy-in of chunk c may start once chunk c - 3 has been computed, and
// each size taken twice on the way up keeps every copy-in behind the
// kernels of the chunks before it.
int grow(int k) { return std::max(k + 1, (4 * k) / 3); }

void chunk_sizes(int BH, int heads_per_chunk, std::vector<int>& out) {
  out.clear();
  if (heads_per_chunk > 0) {
    for (int h0 = 0; h0 < BH; h0 += heads_per_chunk) out.push_back(std::min(heads_per_chunk, BH - h0));
    return;
  }
  const int per = (BH + kDefaultChunks - 1) / kDefaultChunks;
  // up: 1, 1, 2, 2, 3, 3, 4, 4, then growing by grow(); down: the plain
  // grow() ramp, reversed
  std::vector<int> up, down;
  for (int k = 1; k < per; k = grow(k)) {
    up.push_back(k);
    if (k <= 4) up.push_back(k);
  }
  for (int k = 1; k < per; k = grow(k)) down.insert(down.begin(), k);
  auto sum = [](const std::vector<int>& v) {
    int t = 0;
    for (int x : v) t += x;
    return t;
  };
  // the middle: chunks between the ramps' top size and min(per, grow(top));
  // hand the top steps of both ramps to it until such chunks fit
  int mid = 0, n_mid = 0;
  while (true) {
    const int top = std::max(up.empty() ? 0 : up.back(), down.empty() ? 0 : down.front());
    const int cap = top ? std::min(per, grow(top)) : per;
    mid = BH - sum(up) - sum(down);
    n_mid = (mid + cap - 1) / cap;
    if (mid >= std::max(top, 1) && mid / n_mid >= top) break;
    if (up.empty() && down.empty()) break;
    while (!up.empty() && up.back() >= top) up.pop_back();
    while (!down.empty() && down.front() >= top) down.erase(down.begin());
  }
  out = up;
  for (int i = 0; i < n_mid; ++i) out.push_back(mid / n_mid + (i < mid % n_mid ? 1 : 0));
  out.insert(out.end(), down.begin(), down.end());
}

ra_status plan(const ra_problem* p, int heads_per_chunk, HostPlan* hp) {
  ra::Prob P;
  ra_status st = ra::derive_problem(p, &P);
  if (st != RA_OK) return st;
  if (heads_per_chunk < 0) {
    ra::set_error_detail("heads_per_chunk must be >= 0 (0: the library's default)");
    return RA_ERR_INVALID_ARG;
  }
  HostPlan& h = *hp;
  h.BH = P.BH;
  chunk_sizes(P.BH, heads_per_chunk, h.heads);
  h.per = *std::max_element(h.heads.begin(), h.heads.end());
  h.chunk = *p;
  h.chunk.B = 1;
  h.chunk.H = h.per;
  h.head_bytes = (size_t)P.N * ra::D * 2;
  h.ws = ra::align256(ra_workspace_bytes(&h.chunk, 0));
  h.qkv4 = ra::align256(ra_qkv4_bytes(&h.chunk));
  h.io = ra::align256(4 * h.per * h.head_bytes);    // q, k, v, o of one chunk
  h.slot = h.ws + h.qkv4 + h.io;
  h.total = kSlots * h.slot;
  return RA_OK;
}

ra_status cuda_err(cudaError_t e, const char* what) {
  char buf[200];
  snprintf(buf, sizeof(buf), "%s: %s", what, cudaGetErrorString(e));
  cudaGetLastError();
  ra::set_error_detail(buf);
  return RA_ERR_CUDA;
}

// Streams and events of one call, released on every path out of it.
struct Pipeline {
  cudaStream_t in = nullptr, out = nullptr, lane1 = nullptr;
  cudaEvent_t loaded[kSlots] = {}, computed[kSlots] = {}, stored[kSlots] = {};
  cudaEvent_t lane_done[2] = {};
  ~Pipeline() {
    for (int i = 0; i < 2; ++i)
      if (lane_done[i]) cudaEventDestroy(lane_done[i]);
    for (int i = 0; i < kSlots; ++i) {
      if (loaded[i]) cudaEventDestroy(loaded[i]);
      if (computed[i]) cudaEventDestroy(computed[i]);
      if (stored[i]) cudaEventDestroy(stored[i]);
    }
    if (in) cudaStreamDestroy(in);
    if (out) cudaStreamDestroy(out);
    if (lane1) cudaStreamDestroy(lane1);
  }
  cudaError_t create() {
    cudaError_t e = cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&lane1, cudaStreamNonBlocking);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&lane_done[i], cudaEventDisableTiming);
    for (int i = 0; i < kSlots && e == cudaSuccess; ++i) {
      e = cudaEventCreateWithFlags(&loaded[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&computed[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&stored[i], cudaEventDisableTiming);
    }
    return e;
  }
};

}  // namespace

extern "C" {

size_t ra_host_staging_bytes(const ra_problem* p, int heads_per_chunk) {
  HostPlan h;
  return plan(p, heads_per_chunk, &h) == RA_OK ? h.total : 0;
}

int ra_host_chunks(const ra_problem* p, int heads_per_chunk, int* sizes, int max_chunks) {
  HostPlan h;
  if (plan(p, heads_per_chunk, &h) != RA_OK) return -1;
  const int n = (int)h.heads.size();
  if (sizes != nullptr)
    for (int i = 0; i < n && i < max_chunks; ++i) sizes[i] = h.heads[i];
  return n;
}

ra_status ra_int4_attention_host(const ra_problem* p, const void* q, const void* k, const void* v, void* o,
                                 int heads_per_chunk, void* staging, size_t staging_bytes, ra_stream stream) {
  HostPlan h;
  ra_status st = plan(p, heads_per_chunk, &h);
  if (st != RA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) {
    ra::set_error_detail("host q, k, v or o is NULL");
    return RA_ERR_INVALID_ARG;
  }
  if (staging == nullptr || (reinterpret_cast<uintptr_t>(staging) & 255u)) {
    ra::set_error_detail("staging buffer NULL or not 256-byte aligned");
    return RA_ERR_INVALID_ARG;
  }
  if (staging_bytes < h.total) {
    char buf[160];
    snprintf(buf, sizeof(buf), "staging buffer has %zu bytes, needs %zu", staging_bytes, h.total);
    ra::set_error_detail(buf);
    return RA_ERR_WORKSPACE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(staging);
  void* ws[kSlots];
  for (int i = 0; i < kSlots; ++i) ws[i] = base + i * h.slot;

  // Tables and signature of every slot's workspace (synchronises `stream`);
  // the signature does not cover B or H, so each serves every chunk size.
  for (int i = 0; i < kSlots; ++i)
    if ((st = ra_prepare(&h.chunk, ws[i], h.ws, stream)) != RA_OK) return st;

  Pipeline pl;
  cudaError_t e = pl.create();
  if (e != cudaSuccess) return cuda_err(e, "stream/event creation");
  cudaStream_t lane[2] = {s, pl.lane1};

  const char* qh = static_cast<const char*>(q);
  const char* kh = static_cast<const char*>(k);
  const char* vh = static_cast<const char*>(v);
  char* oh = static_cast<char*>(o);
  size_t off = 0;   // first byte of the chunk in every host tensor
  for (size_t c = 0; c < h.heads.size(); ++c) {
    const int sl = (int)(c % kSlots), ln = (int)(c & 1);
    ra_problem cp = h.chunk;
    cp.H = h.heads[c];
    char* slot = base + sl * h.slot;
    ra_qkv4 qkv;
    if ((st = ra_qkv4_bind(&cp, slot + h.ws, h.qkv4, &qkv)) != RA_OK) break;
    const size_t n = (size_t)cp.H * h.head_bytes;
    char* io = slot + h.ws + h.qkv4;
    char *qd = io, *kd = io + n, *vd = io + 2 * n, *od = io + 3 * n;

    // copy-in: the slot is free once chunk c - kSlots has been computed
    if (c >= (size_t)kSlots && (e = cudaStreamWaitEvent(pl.in, pl.computed[sl], 0)) != cudaSuccess) break;
    if ((e = cudaMemcpyAsync(qd, qh + off, n, cudaMemcpyHostToDevice, pl.in)) != cudaSuccess) break;
    if ((e = cudaMemcpyAsync(kd, kh + off, n, cudaMemcpyHostToDevice, pl.in)) != cudaSuccess) break;
    if ((e = cudaMemcpyAsync(vd, vh + off, n, cudaMemcpyHostToDevice, pl.in)) != cudaSuccess) break;
    if ((e = cudaEventRecord(pl.loaded[sl], pl.in)) != cudaSuccess) break;

    // compute on lane c % 2 (after chunk c-2 on the same lane): inputs
    // loaded, and the slot's output read back (chunk c - kSlots)
    if ((e = cudaStreamWaitEvent(lane[ln], pl.loaded[sl], 0)) != cudaSuccess) break;
    if (c >= (size_t)kSlots && (e = cudaStreamWaitEvent(lane[ln], pl.stored[sl], 0)) != cudaSuccess) break;
    if ((st = ra_rotate_quantize_qkv(&cp, qd, kd, vd, &qkv, ws[sl], h.ws, lane[ln])) != RA_OK) break;
    if ((st = ra_int4_attention_fwd(&cp, &qkv, od, ws[sl], h.ws, lane[ln])) != RA_OK) break;
    if ((e = cudaEventRecord(pl.computed[sl], lane[ln])) != cudaSuccess) break;

    // copy-out
    if ((e = cudaStreamWaitEvent(pl.out, pl.computed[sl], 0)) != cudaSuccess) break;
    if ((e = cudaMemcpyAsync(oh + off, od, n, cudaMemcpyDeviceToHost, pl.out)) != cudaSuccess) break;
    if ((e = cudaEventRecord(pl.stored[sl], pl.out)) != cudaSuccess) break;
    off += n;
  }
  // Join the other streams into the caller's stream, then wait for all of it,
  // also on an error path (nothing may still use the staging buffer on return).
  cudaError_t j = cudaEventRecord(pl.loaded[0], pl.in);
  if (j == cudaSuccess) j = cudaStreamWaitEvent(s, pl.loaded[0], 0);
  if (j == cudaSuccess) j = cudaEventRecord(pl.lane_done[1], pl.lane1);
  if (j == cudaSuccess) j = cudaStreamWaitEvent(s, pl.lane_done[1], 0);
  if (j == cudaSuccess) j = cudaEventRecord(pl.stored[0], pl.out);
  if (j == cudaSuccess) j = cudaStreamWaitEvent(s, pl.stored[0], 0);
  cudaError_t w = cudaStreamSynchronize(s);
  if (st != RA_OK) return st;
  if (e != cudaSuccess) return cuda_err(e, "pipeline enqueue");
  if (j != cudaSuccess) return cuda_err(j, "pipeline join");
  if (w != cudaSuccess) return cuda_err(w, "pipeline synchronize");
  for (int i = 0; i < kSlots; ++i)
    if ((st = ra_check_device_error(ws[i], stream)) != RA_OK) return st;
  return RA_OK;
}

}  // extern "C"
