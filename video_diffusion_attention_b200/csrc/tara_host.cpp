// tara_host.cpp -- the forward pass on host buffers: a four-stream copy / compute pipeline.
//
// The B*H (branch, head) planes of Q, K, V, O and LSE are independent, so the call cuts them
// into chunks of consecutive planes and runs, per chunk, host->device copies of its Q, K, V on
// one stream, its attention on device chunk buffers on one of two compute streams, and the
// device->host copies of its O and LSE on a fourth.  Two buffer sets, each with its own
// workspace, alternate between consecutive chunks, and so do the compute streams: the copies of
// one chunk overlap the kernels of its neighbours, and the next chunk's kernel starts on the
// SMs that the current one's last wave leaves idle.  Chunk sizes ramp up 1, 2, 4, ... planes at
// the start and down at the end, so one plane's inputs and one plane's outputs are exposed.
// Everything is ordered after the work already queued on the caller's stream, and the
// caller's stream waits for the last copy.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "forward_internal.h"
#include "param_checks.h"
#include "tara_attn.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kChunkTargetBytes = size_t(1) << 30;   // Q+K+V+O bytes per chunk (~1 GiB)

struct HostPipe {
  bool ready = false;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaStream_t s_comp[2] = {nullptr, nullptr};
  cudaEvent_t ev_start = nullptr, ev_meta = nullptr, ev_done = nullptr;
  cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_comp[2] = {nullptr, nullptr};
  cudaEvent_t ev_out[2] = {nullptr, nullptr};
  void* buf = nullptr;
  size_t buf_bytes = 0;
};

std::mutex g_host_mu;
HostPipe g_pipe[kMaxDevices];

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int pipe_for_device(size_t bytes, HostPipe** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TARA_ERR_CUDA;
  HostPipe& p = g_pipe[dev];
  if (!p.ready) {
    const unsigned f = cudaEventDisableTiming;
    cudaEvent_t* evs[] = {&p.ev_start, &p.ev_meta, &p.ev_done, &p.ev_in[0], &p.ev_in[1],
                          &p.ev_comp[0], &p.ev_comp[1], &p.ev_out[0], &p.ev_out[1]};
    if (cudaStreamCreateWithFlags(&p.s_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&p.s_comp[0], cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&p.s_comp[1], cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&p.s_out, cudaStreamNonBlocking) != cudaSuccess)
      return TARA_ERR_CUDA;
    for (cudaEvent_t* e : evs)
      if (cudaEventCreateWithFlags(e, f) != cudaSuccess) return TARA_ERR_CUDA;
    p.ready = true;
  }
  if (bytes > p.buf_bytes) {
    if (p.buf) {
      cudaFree(p.buf);   // synchronises the device: no earlier call still uses it
      p.buf = nullptr;
      p.buf_bytes = 0;
    }
    if (cudaMalloc(&p.buf, bytes) != cudaSuccess) {
      p.buf = nullptr;
      return TARA_ERR_CUDA;
    }
    p.buf_bytes = bytes;
  }
  *out = &p;
  return TARA_OK;
}

int esize(int dtype) { return dtype == TARA_FP32 ? 4 : 2; }

// Chunk sizes, in planes, of a call over P planes with at most G planes per chunk: 1, 2, 4, ...
// (each step only while both ramps still fit in P), the middle in near-equal chunks of at most
// G, then the ramp reversed.
std::vector<long long> chunk_sizes(long long P, long long G) {
  std::vector<long long> head;
  long long hs = 0;
  for (long long s = 1; s < G && 2 * (hs + s) <= P; s *= 2) {
    head.push_back(s);
    hs += s;
  }
  std::vector<long long> out(head);
  const long long mid = P - 2 * hs;
  if (mid > 0) {
    const long long n = (mid + G - 1) / G;
    for (long long i = 0; i < n; ++i) out.push_back(mid / n + (i < mid % n ? 1 : 0));
  }
  for (auto it = head.rbegin(); it != head.rend(); ++it) out.push_back(*it);
  return out;
}

}  // namespace

extern "C" int tara_attn_forward_host(const tara_tensor* Q, const tara_tensor* K,
                                      const tara_tensor* V, const tara_token_meta* meta,
                                      const tara_params* p, tara_tensor* O, float* LSE,
                                      void* stream_) {
  if (!Q || !K || !V || !meta || !p || !O || !LSE) return TARA_ERR_NULL;
  if (!Q->ptr || !K->ptr || !V->ptr || !O->ptr) return TARA_ERR_NULL;
  if (!meta->seg || !meta->time_s || !meta->pic || !meta->m) return TARA_ERR_NULL;
  const tara_tensor* ts[4] = {Q, K, V, O};
  for (const tara_tensor* t : ts) {
    if (t->dtype != TARA_BF16 && t->dtype != TARA_FP16 && t->dtype != TARA_FP32)
      return TARA_ERR_DTYPE;
    if (t->dtype != Q->dtype) return TARA_ERR_DTYPE;
    if (t->B < 1 || t->H < 1 || t->N < 1 || t->D < 1) return TARA_ERR_SHAPE;
    if (t->B != Q->B || t->H != Q->H || t->N != Q->N || t->D != Q->D) return TARA_ERR_SHAPE;
  }
  if (meta->N != Q->N) return TARA_ERR_SHAPE;
  if (meta->batch_stride < 0 || (meta->batch_stride != 0 && meta->batch_stride < meta->N))
    return TARA_ERR_SHAPE;
  if (Q->dtype == TARA_FP32 ? Q->D > 256 : (Q->D != 64 && Q->D != 128)) return TARA_ERR_HEAD_DIM;
  int rc = tara::check_params(p);
  if (rc != TARA_OK) return rc;
  if (p->qk_int8 && Q->dtype == TARA_FP32) return TARA_ERR_DTYPE;
  if (p->qk_int8 && Q->D != 128) return TARA_ERR_HEAD_DIM;
  if (p->n_extra_bindings > 0 && !meta->extra_m) return TARA_ERR_NULL;

  const int B = Q->B, H = Q->H, N = Q->N, D = Q->D;
  const size_t es = (size_t)esize(Q->dtype);
  const size_t plane = (size_t)N * D * es;           // one (branch, head) plane of Q, K, V or O
  const size_t lse_plane = (size_t)N * sizeof(float);
  const long long P = (long long)B * H;
  // chunk: G consecutive planes, never across a branch when each branch has its own metadata
  long long G = (long long)(kChunkTargetBytes / (4 * plane));
  if (G < 1) G = 1;
  if (G > P) G = P;
  if (meta->batch_stride != 0 && G > H) G = H;
  const bool strided = meta->batch_stride != 0;

  // metadata arrays: one set, or B sets batch_stride apart
  const long long nsets = strided ? B : 1;
  const size_t m_len = (size_t)((nsets - 1) * meta->batch_stride + N);
  const int nx = p->n_extra_bindings;
  const size_t x_len = nx > 0 ? (size_t)(nx - 1) * (size_t)meta->extra_m_stride + m_len : 0;
  if (nx > 0 && (size_t)meta->extra_m_stride < m_len) return TARA_ERR_SHAPE;

  const size_t off_time = round_up(m_len, 256);
  const size_t off_pic = off_time + round_up(m_len * 4, 256);
  const size_t off_m = off_pic + round_up(m_len, 256);
  const size_t off_x = off_m + round_up(m_len * 4, 256);
  const size_t meta_bytes = off_x + round_up(x_len * 4, 256);
  const size_t chunk_bytes = round_up((size_t)G * plane, 256);
  const size_t chunk_lse = round_up((size_t)G * lse_plane, 256);
  // workspace of the largest chunk (B = 1, G planes, one metadata set)
  tara_tensor tg = *Q;
  tg.B = 1;
  tg.H = (int32_t)G;
  tara_token_meta mg = *meta;
  mg.batch_stride = 0;
  const size_t ws_bytes = round_up(tara::forward_workspace_bytes(&tg, &mg, p), 256);
  // Q, K, V, O, LSE and the workspace of one chunk
  const size_t set_bytes = 4 * chunk_bytes + chunk_lse + ws_bytes;

  std::lock_guard<std::mutex> lock(g_host_mu);
  HostPipe* pp = nullptr;
  rc = pipe_for_device(meta_bytes + 2 * set_bytes, &pp);
  if (rc != TARA_OK) return rc;
  HostPipe& pipe = *pp;
  cudaStream_t user = static_cast<cudaStream_t>(stream_);
  char* base = static_cast<char*>(pipe.buf);
  // a kernel-event pair pending for this thread would bracket a chunk, not the call: drop it
  tara_set_kernel_events(nullptr, nullptr);

  // the previous call's last kernels and copies still use the buffer sets (ev_done is its end;
  // a never-recorded event is complete)
  bool cuda_ok = cudaEventRecord(pipe.ev_start, user) == cudaSuccess &&
                 cudaStreamWaitEvent(pipe.s_out, pipe.ev_start, 0) == cudaSuccess;
  cudaStream_t waiters[3] = {pipe.s_in, pipe.s_comp[0], pipe.s_comp[1]};
  for (cudaStream_t w : waiters)
    cuda_ok = cuda_ok && cudaStreamWaitEvent(w, pipe.ev_done, 0) == cudaSuccess &&
              cudaStreamWaitEvent(w, pipe.ev_start, 0) == cudaSuccess;
  // metadata in once
  cuda_ok = cuda_ok &&
            cudaMemcpyAsync(base, meta->seg, m_len, cudaMemcpyHostToDevice, pipe.s_in) == cudaSuccess &&
            cudaMemcpyAsync(base + off_time, meta->time_s, m_len * 4, cudaMemcpyHostToDevice, pipe.s_in) == cudaSuccess &&
            cudaMemcpyAsync(base + off_pic, meta->pic, m_len, cudaMemcpyHostToDevice, pipe.s_in) == cudaSuccess &&
            cudaMemcpyAsync(base + off_m, meta->m, m_len * 4, cudaMemcpyHostToDevice, pipe.s_in) == cudaSuccess &&
            (x_len == 0 || cudaMemcpyAsync(base + off_x, meta->extra_m, x_len * 4,
                                           cudaMemcpyHostToDevice, pipe.s_in) == cudaSuccess) &&
            cudaEventRecord(pipe.ev_meta, pipe.s_in) == cudaSuccess &&
            cudaStreamWaitEvent(pipe.s_comp[0], pipe.ev_meta, 0) == cudaSuccess &&
            cudaStreamWaitEvent(pipe.s_comp[1], pipe.ev_meta, 0) == cudaSuccess;

  const char* hq = static_cast<const char*>(Q->ptr);
  const char* hk = static_cast<const char*>(K->ptr);
  const char* hv = static_cast<const char*>(V->ptr);
  char* ho = static_cast<char*>(O->ptr);
  char* hl = reinterpret_cast<char*>(LSE);
  const std::vector<long long> sizes = chunk_sizes(P, G);
  long long c = 0, p0 = 0;
  for (size_t si = 0; si < sizes.size() && cuda_ok && rc == TARA_OK; ++si) {
    for (long long want = sizes[si]; want > 0 && cuda_ok && rc == TARA_OK; ++c) {
      long long g = want;
      if (strided && (p0 / H) != ((p0 + g - 1) / H)) g = (p0 / H + 1) * H - p0;   // stay in branch
      want -= g;
      const int b = (int)(p0 / H);
      const int k = (int)(c & 1);
      cudaStream_t comp = pipe.s_comp[k];
      char* cb = base + meta_bytes + (size_t)k * set_bytes;
      char *dq = cb, *dk = cb + chunk_bytes, *dv = cb + 2 * chunk_bytes, *dout = cb + 3 * chunk_bytes;
      float* dl = reinterpret_cast<float*>(cb + 4 * chunk_bytes);
      void* dws = cb + 4 * chunk_bytes + chunk_lse;
      const size_t bytes = (size_t)g * plane, off = (size_t)p0 * plane;
      // inputs: the chunk two back must have finished reading this buffer set
      if (c >= 2) cuda_ok = cudaStreamWaitEvent(pipe.s_in, pipe.ev_comp[k], 0) == cudaSuccess;
      cuda_ok = cuda_ok &&
                cudaMemcpyAsync(dq, hq + off, bytes, cudaMemcpyHostToDevice, pipe.s_in) == cudaSuccess &&
                cudaMemcpyAsync(dk, hk + off, bytes, cudaMemcpyHostToDevice, pipe.s_in) == cudaSuccess &&
                cudaMemcpyAsync(dv, hv + off, bytes, cudaMemcpyHostToDevice, pipe.s_in) == cudaSuccess &&
                cudaEventRecord(pipe.ev_in[k], pipe.s_in) == cudaSuccess &&
                cudaStreamWaitEvent(comp, pipe.ev_in[k], 0) == cudaSuccess;
      // compute: the outputs of the chunk two back must have been copied out (its kernel ran
      // on the same stream, so the buffer set's workspace is free as well)
      if (cuda_ok && c >= 2) cuda_ok = cudaStreamWaitEvent(comp, pipe.ev_out[k], 0) == cudaSuccess;
      if (!cuda_ok) break;
      tara_tensor tq = *Q, tk = *K, tv = *V, to = *O;
      tq.ptr = dq;
      tk.ptr = dk;
      tv.ptr = dv;
      to.ptr = dout;
      tq.B = tk.B = tv.B = to.B = 1;
      tq.H = tk.H = tv.H = to.H = (int32_t)g;
      tara_token_meta dm = *meta;
      const size_t mo = strided ? (size_t)b * (size_t)meta->batch_stride : 0;
      dm.seg = reinterpret_cast<const uint8_t*>(base) + mo;
      dm.time_s = reinterpret_cast<const float*>(base + off_time) + mo;
      dm.pic = reinterpret_cast<const uint8_t*>(base + off_pic) + mo;
      dm.m = reinterpret_cast<const float*>(base + off_m) + mo;
      dm.extra_m = nx > 0 ? reinterpret_cast<const float*>(base + off_x) + mo : nullptr;
      dm.batch_stride = 0;
      rc = tara::forward_with_workspace(&tq, &tk, &tv, &dm, p, &to, dl, dws, ws_bytes, comp, p0);
      if (rc != TARA_OK) break;
      cuda_ok = cudaEventRecord(pipe.ev_comp[k], comp) == cudaSuccess &&
                cudaStreamWaitEvent(pipe.s_out, pipe.ev_comp[k], 0) == cudaSuccess &&
                cudaMemcpyAsync(ho + off, dout, bytes, cudaMemcpyDeviceToHost, pipe.s_out) == cudaSuccess &&
                cudaMemcpyAsync(hl + (size_t)p0 * lse_plane, dl, (size_t)g * lse_plane,
                                cudaMemcpyDeviceToHost, pipe.s_out) == cudaSuccess &&
                cudaEventRecord(pipe.ev_out[k], pipe.s_out) == cudaSuccess;
      p0 += g;
    }
  }
  // the caller's stream waits for everything queued above on all four streams, whatever
  // happened; ev_done ends on s_out after s_in and both compute streams have drained into it
  bool join_ok = true;
  for (cudaStream_t w : waiters)
    join_ok = join_ok && cudaEventRecord(pipe.ev_done, w) == cudaSuccess &&
              cudaStreamWaitEvent(pipe.s_out, pipe.ev_done, 0) == cudaSuccess;
  join_ok = join_ok && cudaEventRecord(pipe.ev_done, pipe.s_out) == cudaSuccess &&
            cudaStreamWaitEvent(user, pipe.ev_done, 0) == cudaSuccess;
  if (rc != TARA_OK) return rc;
  return (cuda_ok && join_ok) ? TARA_OK : TARA_ERR_CUDA;
}
