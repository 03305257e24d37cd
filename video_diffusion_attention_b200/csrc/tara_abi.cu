// tara_abi.cu -- the C ABI of the library: argument checks, the per-device workspace, tensor
// maps, and the launches of the tile-summary, tensor-core and CUDA-core kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "tara_attn.h"
#include "forward_internal.h"
#include "param_checks.h"
#include "attn_pair.cuh"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "quant_int8.cuh"
#include "target_mask.cuh"
#include "tile_summary.cuh"

namespace tara {
namespace {

// Set by any kernel that gave up on a bounded wait; read and cleared by tara_device_status.
__device__ int g_device_status;

constexpr int kMaxDevices = 64;

struct DeviceState {
  void* ws = nullptr;           // tile summaries + per-key records
  size_t ws_bytes = 0;
  int* status = nullptr;        // device address of g_device_status
  bool tc_attr_set[2][2] = {{false, false}, {false, false}};   // [bf16][D==128]
  bool tc_q8_attr_set[2] = {false, false};                     // [bf16], D = 128
  bool pair_attr_set[2] = {false, false};                      // [bf16], D = 128
  bool simt_attr_set = false;
  // recorded on a call's stream after its last workspace reader; the next call's stream waits
  // on it before rewriting the workspace, so calls on different streams serialise on the GPU
  cudaEvent_t ws_free = nullptr;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

// Event pair set by tara_set_kernel_events for the calling thread's next forward call.
thread_local cudaEvent_t t_ev_start = nullptr, t_ev_stop = nullptr;

int record_start(cudaStream_t stream) {
  if (t_ev_start && cudaEventRecord(t_ev_start, stream) != cudaSuccess) return TARA_ERR_CUDA;
  return TARA_OK;
}
int record_stop(cudaStream_t stream) {
  cudaEvent_t ev = t_ev_stop;
  t_ev_start = t_ev_stop = nullptr;
  if (ev && cudaEventRecord(ev, stream) != cudaSuccess) return TARA_ERR_CUDA;
  return TARA_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

// Resolves the driver's tensor-map encoder once per process; both forward entry points call
// this under different mutexes, so the lookup itself is guarded by its own once-flag.
int get_encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && fn != nullptr)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode ? TARA_OK : TARA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

BiasParams make_bias_params(const tara_params* p, int D) {
  BiasParams bp;
  std::memset(&bp, 0, sizeof(bp));
  bp.window = p->window;
  bp.inv_falloff = (float)(1.0 / (double)p->falloff);
  bp.strength = p->strength;
  bp.cap = p->cap;
  const double scale = p->softmax_scale > 0.0f ? (double)p->softmax_scale
                                                : 1.0 / std::sqrt((double)D);
  bp.scale = (float)scale;
  bp.scale_log2 = (float)(scale * 1.4426950408889634);
  bp.lng_nz = 0;
  for (int i = 1; i <= 9; ++i) {
    bp.lng[i] = (float)std::log((double)p->gain[i - 1]);
    if (bp.lng[i] != 0.0f) bp.lng_nz |= 1u << i;
  }
  bp.n_extra = p->n_extra_bindings;
  for (int k = 0; k < p->n_extra_bindings; ++k)
    for (int i = 1; i <= 9; ++i) {
      bp.lng_x[k][i] = (float)std::log((double)p->extra_gain[k][i - 1]);
      if (bp.lng_x[k][i] != 0.0f) bp.lng_nz |= 1u << i;
    }
  return bp;
}

// Tensor map of a 16-bit [B*H][N][D] tensor: boxes of 64 head-dim columns (one 128-byte
// swizzle panel) by box_rows tokens.
int encode_qkv_map(CUtensorMap* map, const tara_tensor* t, uint32_t box_rows = kTile) {
  const CUtensorMapDataType dt =
      t->dtype == TARA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t dims[3] = {(cuuint64_t)t->D, (cuuint64_t)t->N,
                              (cuuint64_t)t->B * (cuuint64_t)t->H};
  const cuuint64_t strides[2] = {(cuuint64_t)t->D * 2, (cuuint64_t)t->N * (cuuint64_t)t->D * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, dt, 3, t->ptr, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TARA_OK : TARA_ERR_CUDA;
}

// Tensor map of 8-bit codes [B*H][N][D] (D = 128): one 128-byte swizzle panel per row.
int encode_q8_map(CUtensorMap* map, const void* codes, int BH, int N, int D) {
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)D, (cuuint64_t)N * (cuuint64_t)D};
  const cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)kTile, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(codes), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TARA_OK : TARA_ERR_CUDA;
}

// The tensor-core kernel's setmaxnreg split assumes ptxas gave it exactly kTcLaunchRegs
// registers per thread (the pool the raise draws on); any other count is refused here rather
// than launched.
template <typename F>
int tc_register_check(F* kernel) {
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return TARA_ERR_CUDA;
  return fa.numRegs == kTcLaunchRegs ? TARA_OK : TARA_ERR_CUDA;
}

// Quantises Q per token and K per 128-token block (quant_int8.cuh).
int launch_quant(const tara_tensor* Q, const tara_tensor* K, int8_t* qc, float* qs, int8_t* kc,
                 float* ks, cudaStream_t stream) {
  const bool bf16 = Q->dtype == TARA_BF16;
  const int BH = Q->B * Q->H, N = Q->N, D = Q->D;
  const long long rows = (long long)BH * N;
  // rows per CTA: its warps x (32 / (D/8)) rows per load x kQRowsUnroll loads
  const long long q_rows_cta = (long long)(kQ8Threads / 32) * (256 / D) * kQRowsUnroll;
  const unsigned qgrid = (unsigned)((rows + q_rows_cta - 1) / q_rows_cta);
  const dim3 kgrid((unsigned)((N + kQ8Block - 1) / kQ8Block), (unsigned)BH);
  const int nb = (N + kQ8Block - 1) / kQ8Block;
  const uint16_t* q = static_cast<const uint16_t*>(Q->ptr);
  const uint16_t* k = static_cast<const uint16_t*>(K->ptr);
  if (D == 128) {
    if (bf16) {
      quant_q_kernel<true, 128><<<qgrid, kQ8Threads, 0, stream>>>(q, rows, qc, qs);
      quant_k_kernel<true, 128><<<kgrid, kQ8Threads, 0, stream>>>(k, N, nb, kc, ks);
    } else {
      quant_q_kernel<false, 128><<<qgrid, kQ8Threads, 0, stream>>>(q, rows, qc, qs);
      quant_k_kernel<false, 128><<<kgrid, kQ8Threads, 0, stream>>>(k, N, nb, kc, ks);
    }
  } else {
    if (bf16) {
      quant_q_kernel<true, 64><<<qgrid, kQ8Threads, 0, stream>>>(q, rows, qc, qs);
      quant_k_kernel<true, 64><<<kgrid, kQ8Threads, 0, stream>>>(k, N, nb, kc, ks);
    } else {
      quant_q_kernel<false, 64><<<qgrid, kQ8Threads, 0, stream>>>(q, rows, qc, qs);
      quant_k_kernel<false, 64><<<kgrid, kQ8Threads, 0, stream>>>(k, N, nb, kc, ks);
    }
  }
  return cudaGetLastError() == cudaSuccess ? TARA_OK : TARA_ERR_CUDA;
}

// Returns the device's state with a workspace of at least `bytes` (grown with cudaMalloc).
int device_state(size_t bytes, DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TARA_ERR_CUDA;
  DeviceState& st = g_dev[dev];
  if (st.status == nullptr) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_device_status) != cudaSuccess) return TARA_ERR_CUDA;
    st.status = static_cast<int*>(addr);
  }
  if (bytes > st.ws_bytes) {
    if (st.ws) {
      cudaFree(st.ws);   // synchronises the device: no earlier call still reads it
      st.ws = nullptr;
      st.ws_bytes = 0;
    }
    if (cudaMalloc(&st.ws, bytes) != cudaSuccess) {
      st.ws = nullptr;
      return TARA_ERR_CUDA;
    }
    st.ws_bytes = bytes;
  }
  *out = &st;
  return TARA_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Self-test of the bounded-wait machinery: one warp waits on an mbarrier phase; with
// arrive == 0 nothing ever arrives, so the wait must give up after limit_ns and set the
// device status word exactly as an attention kernel does.
__global__ void wait_selftest_kernel(int* status, uint64_t limit_ns, int arrive) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (arrive) mbar_arrive(&bar);
    if (!mbar_wait(&bar, 0, &abort_flag, limit_ns)) atomicExch(status, 1);
  }
}

template <bool kBF16, int D, bool kQ8 = false>
int launch_tc(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
              const TcArgs& a, int B, int H, int ntiles, cudaStream_t stream, DeviceState* st) {
  constexpr int smem = TcShape<D, kQ8>::kSmemBytes;
  bool& attr = kQ8 ? st->tc_q8_attr_set[kBF16 ? 1 : 0]
                   : st->tc_attr_set[kBF16 ? 1 : 0][D == 128 ? 1 : 0];
  if (!attr) {
    if (tc_register_check(attn_tc_kernel<kBF16, D, kQ8>) != TARA_OK) return TARA_ERR_CUDA;
    if (cudaFuncSetAttribute(attn_tc_kernel<kBF16, D, kQ8>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return TARA_ERR_CUDA;
    attr = true;
  }
  dim3 grid((unsigned)((ntiles + 1) / 2), (unsigned)H, (unsigned)B);
  if (record_start(stream) != TARA_OK) return TARA_ERR_CUDA;
  attn_tc_kernel<kBF16, D, kQ8><<<grid, kTcThreads, smem, stream>>>(mq, mk, mv, a);
  if (cudaGetLastError() != cudaSuccess) return TARA_ERR_CUDA;
  return record_stop(stream);
}

// Head dim 128, 16-bit Q/K: the SM-pair kernel.  Two CTAs per four query tiles; the K map
// has 64-row boxes (each CTA of a pair loads half of every key tile).  `attr` caches the
// one-time attribute set-up (nullptr: set it on every call).
template <bool kBF16>
int launch_pair(const tara_tensor* Q, const tara_tensor* K, const tara_tensor* V,
                const TcArgs& a, int B, int H, int ntiles, cudaStream_t stream, bool* attr) {
  constexpr int smem = PairShape::kSmemBytes;
  if (!attr || !*attr) {
    if (tc_register_check(attn_pair_kernel<kBF16>) != TARA_OK) return TARA_ERR_CUDA;
    if (cudaFuncSetAttribute(attn_pair_kernel<kBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return TARA_ERR_CUDA;
    if (attr) *attr = true;
  }
  CUtensorMap mq, mk, mv;
  if (encode_qkv_map(&mq, Q) != TARA_OK || encode_qkv_map(&mk, K, 64) != TARA_OK ||
      encode_qkv_map(&mv, V) != TARA_OK)
    return TARA_ERR_CUDA;
  // persistent: one cluster per SM pair (at most one per work item), each walking the
  // (branch, head, 4-query-tile) items in head-major order
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return TARA_ERR_CUDA;
  const long long items = (long long)B * H * ((ntiles + kPairTiles - 1) / kPairTiles);
  const long long clusters = std::min<long long>(items, std::max(1, sms / 2));
  dim3 grid((unsigned)(2 * clusters), 1, 1);
  // the key order flips every (SMs / 2) items: with a full grid, every round of concurrent
  // items walks the keys the opposite way to the round before and starts on the key tiles
  // that round read last, which are still in L2.  The span depends on the device only, so a
  // plane's result does not depend on how many planes share the call.
  const long long item_base = a.plane_base * ((ntiles + kPairTiles - 1) / kPairTiles);
  if (item_base + items > 0x7fffffffLL) return TARA_ERR_TOO_LARGE;
  TcArgs ap = a;
  ap.item_base = (int)item_base;
  ap.order_span = std::max(1, sms / 2);
  if (record_start(stream) != TARA_OK) return TARA_ERR_CUDA;
  attn_pair_kernel<kBF16><<<grid, kTcThreads, smem, stream>>>(mq, mk, mv, ap);
  if (cudaGetLastError() != cudaSuccess) return TARA_ERR_CUDA;
  return record_stop(stream);
}

// Kernel arguments shared by the workspace and the scratch-array entry points.
TcArgs make_tc_args(const tara_token_meta* meta, tara_tensor* O, float* LSE, TileRec* recs,
                    float4* keyinfo, int N, int H, int ntiles, int* status,
                    const BiasParams& bp, const float* q_scale, const float* k_scale) {
  TcArgs a;
  a.O = O->ptr;
  a.LSE = LSE;
  a.seg = meta->seg;
  a.time_s = meta->time_s;
  a.m = meta->m;
  a.recs = recs;
  a.keyinfo = keyinfo;
  const long long nsets = meta->batch_stride != 0 ? O->B : 1;
  a.recs_desc = recs + nsets * ntiles;
  a.keyinfo_desc = keyinfo + nsets * ntiles * kTile;
  a.meta_stride = (long long)meta->batch_stride;
  a.N = N;
  a.H = H;
  a.ntiles = ntiles;
  a.B = O->B;
  a.per_branch_meta = meta->batch_stride != 0 ? 1 : 0;
  a.status = status;
  a.bp = bp;
  a.xm = ExtraMasks{meta->extra_m, (long long)meta->extra_m_stride};
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.plane_base = 0;
  a.item_base = 0;
  a.order_span = 1;
  return a;
}

int validate(const tara_tensor* Q, const tara_tensor* K, const tara_tensor* V,
             const tara_token_meta* meta, const tara_params* p, const tara_tensor* O,
             const float* LSE) {
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
  if (Q->dtype == TARA_FP32) {
    if (Q->D > kSimtMaxD) return TARA_ERR_HEAD_DIM;
  } else {
    if (Q->D != 64 && Q->D != 128) return TARA_ERR_HEAD_DIM;
  }
  if (Q->B > 65535 || Q->H > 65535) return TARA_ERR_TOO_LARGE;
  if ((long long)Q->B * Q->H > 0x7fffffffLL) return TARA_ERR_TOO_LARGE;
  // the persistent kernel numbers its work items (planes x groups of four query tiles) in int
  if ((long long)Q->B * Q->H * ((((long long)Q->N + kTile - 1) / kTile + 3) / 4) > 0x7fffffffLL)
    return TARA_ERR_TOO_LARGE;
  for (const tara_tensor* t : ts)
    if (!aligned16(t->ptr)) return TARA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(LSE) & 3u) != 0) return TARA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(meta->time_s) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(meta->m) & 3u) != 0)
    return TARA_ERR_ALIGN;
  int rc = check_params(p);
  if (rc != TARA_OK) return rc;
  if (p->qk_int8) {
    if (Q->dtype == TARA_FP32) return TARA_ERR_DTYPE;
    if (Q->D != 128) return TARA_ERR_HEAD_DIM;
  }
  if (p->n_extra_bindings == 0) return TARA_OK;
  // masks of the extra bindings: one array per binding, each as long as m
  if (!meta->extra_m) return TARA_ERR_NULL;
  const long long nsets = meta->batch_stride != 0 ? Q->B : 1;
  const long long m_len = (nsets - 1) * (long long)meta->batch_stride + meta->N;
  if (meta->extra_m_stride < m_len) return TARA_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(meta->extra_m) & 3u) != 0) return TARA_ERR_ALIGN;
  return TARA_OK;
}

// Workspace of one tensor-core forward call: tile records and per-key records of every
// metadata set, in ascending and in descending tile order (tile_summary.cuh), then (qk_int8
// only) the 8-bit copies of Q and K and their scales.
struct WsLayout {
  int nsets;
  size_t rec, key, code, qs, ks, total;
};

WsLayout ws_layout(const tara_tensor* Q, const tara_token_meta* meta, const tara_params* p) {
  WsLayout L;
  const int B = Q->B, H = Q->H, N = Q->N, D = Q->D;
  const int ntiles = (N + kTile - 1) / kTile;
  L.nsets = meta->batch_stride != 0 ? B : 1;
  L.rec = round_up(2 * (size_t)L.nsets * ntiles * sizeof(TileRec), 256);
  L.key = round_up(2 * (size_t)L.nsets * ntiles * kTile * sizeof(float4), 256);
  const bool q8 = p->qk_int8 != 0;
  L.code = q8 ? round_up((size_t)B * H * N * D, 256) : 0;
  L.qs = q8 ? round_up((size_t)B * H * N * sizeof(float), 256) : 0;
  L.ks = q8 ? round_up((size_t)B * H * ntiles * sizeof(float), 256) : 0;
  L.total = Q->dtype == TARA_FP32 ? 0 : L.rec + L.key + 2 * L.code + L.qs + L.ks;
  return L;
}

// The forward pass after argument checks, with g_mu held.  ws_ext == nullptr: the device's
// shared workspace, ordered against every other call through ws_free.  Otherwise the caller's
// workspace of ws_ext_bytes (at least ws_layout(...).total of the shape), which the caller orders.
// plane_base: index of plane 0 within a larger call these planes were cut from (0 otherwise).
int forward_locked(const tara_tensor* Q, const tara_tensor* K, const tara_tensor* V,
                   const tara_token_meta* meta, const tara_params* p, tara_tensor* O, float* LSE,
                   cudaStream_t stream, void* ws_ext, size_t ws_ext_bytes, long long plane_base) {
  int rc = TARA_OK;
  const int B = Q->B, H = Q->H, N = Q->N, D = Q->D;
  const BiasParams bp = make_bias_params(p, D);

  if (Q->dtype == TARA_FP32) {
    DeviceState* st = nullptr;
    if ((rc = device_state(0, &st)) != TARA_OK) return rc;
    const size_t smem = (size_t)(2 * kSimtChunk * (D + 1) + kSimtRows * D) * sizeof(float);
    if (!st->simt_attr_set) {
      if (cudaFuncSetAttribute(attn_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)((2 * kSimtChunk * (kSimtMaxD + 1) + kSimtRows * kSimtMaxD) *
                                     sizeof(float))) != cudaSuccess)
        return TARA_ERR_CUDA;
      st->simt_attr_set = true;
    }
    dim3 grid((unsigned)((N + kSimtRows - 1) / kSimtRows), (unsigned)H, (unsigned)B);
    if (record_start(stream) != TARA_OK) return TARA_ERR_CUDA;
    attn_simt_kernel<<<grid, kSimtRows * 32, smem, stream>>>(
        static_cast<const float*>(Q->ptr), static_cast<const float*>(K->ptr),
        static_cast<const float*>(V->ptr), static_cast<float*>(O->ptr), LSE, meta->seg,
        meta->time_s, meta->pic, meta->m, (long long)meta->batch_stride, H, N, D, bp,
        ExtraMasks{meta->extra_m, (long long)meta->extra_m_stride}, st->status);
    if (cudaGetLastError() != cudaSuccess) return TARA_ERR_CUDA;
    return record_stop(stream);
  }

  if ((rc = get_encode_fn()) != TARA_OK) return rc;
  const int ntiles = (N + kTile - 1) / kTile;
  const WsLayout L = ws_layout(Q, meta, p);
  const bool q8 = p->qk_int8 != 0;
  DeviceState* st = nullptr;
  if ((rc = device_state(ws_ext ? 0 : L.total, &st)) != TARA_OK) return rc;
  if (ws_ext && ws_ext_bytes < L.total) return TARA_ERR_TOO_LARGE;
  char* ws = static_cast<char*>(ws_ext ? ws_ext : st->ws);
  TileRec* recs = reinterpret_cast<TileRec*>(ws);
  float4* keyinfo = reinterpret_cast<float4*>(ws + L.rec);
  int8_t* qc = reinterpret_cast<int8_t*>(ws + L.rec + L.key);
  int8_t* kc = qc + L.code;
  float* qs = reinterpret_cast<float*>(ws + L.rec + L.key + 2 * L.code);
  float* ks = reinterpret_cast<float*>(ws + L.rec + L.key + 2 * L.code + L.qs);

  // wait for the previous call's kernels to finish reading the shared workspace (not while the
  // stream is being captured: a captured wait on an event recorded outside the graph is not
  // allowed; a caller-owned workspace is ordered by its owner)
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return TARA_ERR_CUDA;
  const bool order_ws = cap == cudaStreamCaptureStatusNone && ws_ext == nullptr;
  if (order_ws) {
    if (!st->ws_free && cudaEventCreateWithFlags(&st->ws_free, cudaEventDisableTiming) != cudaSuccess)
      return TARA_ERR_CUDA;
    if (cudaStreamWaitEvent(stream, st->ws_free, 0) != cudaSuccess) return TARA_ERR_CUDA;
  }

  CUtensorMap mq, mk, mv;
  if (q8) {
    if (encode_q8_map(&mq, qc, B * H, N, D) != TARA_OK ||
        encode_q8_map(&mk, kc, B * H, N, D) != TARA_OK || encode_qkv_map(&mv, V) != TARA_OK)
      return TARA_ERR_CUDA;
    if ((rc = launch_quant(Q, K, qc, qs, kc, ks, stream)) != TARA_OK) return rc;
  } else if (encode_qkv_map(&mq, Q) != TARA_OK || encode_qkv_map(&mk, K) != TARA_OK ||
             encode_qkv_map(&mv, V) != TARA_OK) {
    return TARA_ERR_CUDA;
  }

  tile_summary_kernel<<<dim3((unsigned)ntiles, (unsigned)L.nsets), 128, 0, stream>>>(
      meta->seg, meta->time_s, meta->pic, N, (long long)meta->batch_stride, ntiles, bp, recs,
      keyinfo, st->status);
  if (cudaGetLastError() != cudaSuccess) return TARA_ERR_CUDA;

  TcArgs a = make_tc_args(meta, O, LSE, recs, keyinfo, N, H, ntiles, st->status, bp, qs, ks);
  a.plane_base = plane_base;
  const bool bf16 = Q->dtype == TARA_BF16;
  if (q8)
    rc = bf16 ? launch_tc<true, 128, true>(mq, mk, mv, a, B, H, ntiles, stream, st)
              : launch_tc<false, 128, true>(mq, mk, mv, a, B, H, ntiles, stream, st);
  else if (D == 128)
    rc = bf16 ? launch_pair<true>(Q, K, V, a, B, H, ntiles, stream, &st->pair_attr_set[1])
              : launch_pair<false>(Q, K, V, a, B, H, ntiles, stream, &st->pair_attr_set[0]);
  else
    rc = bf16 ? launch_tc<true, 64>(mq, mk, mv, a, B, H, ntiles, stream, st)
              : launch_tc<false, 64>(mq, mk, mv, a, B, H, ntiles, stream, st);
  if (rc == TARA_OK && order_ws && cudaEventRecord(st->ws_free, stream) != cudaSuccess)
    return TARA_ERR_CUDA;
  return rc;
}

}  // namespace

size_t forward_workspace_bytes(const tara_tensor* Q, const tara_token_meta* meta,
                               const tara_params* p) {
  return ws_layout(Q, meta, p).total;
}

int forward_with_workspace(const tara_tensor* Q, const tara_tensor* K, const tara_tensor* V,
                           const tara_token_meta* meta, const tara_params* p, tara_tensor* O,
                           float* LSE, void* ws, size_t ws_bytes, void* stream,
                           long long plane_base) {
  int rc = validate(Q, K, V, meta, p, O, LSE);
  if (plane_base < 0) return TARA_ERR_SHAPE;
  if (rc != TARA_OK) return rc;
  if (Q->dtype != TARA_FP32 && !ws) return TARA_ERR_NULL;
  if (!aligned16(ws)) return TARA_ERR_ALIGN;
  std::lock_guard<std::mutex> lock(g_mu);
  return forward_locked(Q, K, V, meta, p, O, LSE, static_cast<cudaStream_t>(stream), ws, ws_bytes,
                        plane_base);
}

}  // namespace tara

using namespace tara;

extern "C" {

void tara_default_params(tara_params* p) {
  if (!p) return;
  p->window = 0.20f;
  p->falloff = 0.25f;
  p->strength = 2.0f;
  p->cap = 6.0f;
  for (int i = 0; i < 9; ++i) p->gain[i] = 1.0f;
  p->softmax_scale = 0.0f;
  p->n_extra_bindings = 0;
  for (int k = 0; k < TARA_MAX_EXTRA_BINDINGS; ++k)
    for (int i = 0; i < 9; ++i) p->extra_gain[k][i] = 1.0f;
  p->qk_int8 = 0;
}

const char* tara_status_string(int s) {
  switch (s) {
    case TARA_OK: return "ok";
    case TARA_ERR_NULL: return "null pointer";
    case TARA_ERR_SHAPE: return "inconsistent or invalid shape";
    case TARA_ERR_DTYPE: return "invalid or mismatched dtype";
    case TARA_ERR_HEAD_DIM: return "unsupported head dimension";
    case TARA_ERR_PARAM: return "rule parameter out of domain";
    case TARA_ERR_ALIGN: return "misaligned pointer";
    case TARA_ERR_SEGMENT: return "invalid segment description";
    case TARA_ERR_CAPACITY: return "output length does not match the segments";
    case TARA_ERR_CUDA: return "CUDA call failed";
    case TARA_ERR_DEVICE_TIMEOUT: return "a kernel gave up on a bounded wait";
    case TARA_ERR_TOO_LARGE: return "size too large";
    case TARA_ERR_MASK_LENGTH: return "mask is neither one frame nor the prepared shot length";
    case TARA_ERR_DEBUG_CHECK: return "a device-side check of the debug build failed";
    default: return "unknown status";
  }
}

int tara_attn_forward(const tara_tensor* Q, const tara_tensor* K, const tara_tensor* V,
                      const tara_token_meta* meta, const tara_params* p, tara_tensor* O,
                      float* LSE, void* stream_) {
  int rc = validate(Q, K, V, meta, p, O, LSE);
  if (rc != TARA_OK) return rc;
  std::lock_guard<std::mutex> lock(g_mu);
  return forward_locked(Q, K, V, meta, p, O, LSE, static_cast<cudaStream_t>(stream_), nullptr, 0, 0);
}

int tara_quantize_qk_int8(const tara_tensor* Q, const tara_tensor* K, int8_t* q_codes,
                          float* q_scale, int8_t* k_codes, float* k_scale, void* stream) {
  if (!Q || !K || !q_codes || !q_scale || !k_codes || !k_scale) return TARA_ERR_NULL;
  if (!Q->ptr || !K->ptr) return TARA_ERR_NULL;
  if (Q->dtype != TARA_BF16 && Q->dtype != TARA_FP16) return TARA_ERR_DTYPE;
  if (K->dtype != Q->dtype) return TARA_ERR_DTYPE;
  if (Q->B < 1 || Q->H < 1 || Q->N < 1 || Q->D < 1) return TARA_ERR_SHAPE;
  if (K->B != Q->B || K->H != Q->H || K->N != Q->N || K->D != Q->D) return TARA_ERR_SHAPE;
  if (Q->D != 64 && Q->D != 128) return TARA_ERR_HEAD_DIM;
  if ((long long)Q->B * Q->H > 65535) return TARA_ERR_TOO_LARGE;
  if (!aligned16(Q->ptr) || !aligned16(K->ptr) || !aligned16(q_codes) || !aligned16(k_codes))
    return TARA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(q_scale) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(k_scale) & 3u) != 0)
    return TARA_ERR_ALIGN;
  return launch_quant(Q, K, q_codes, q_scale, k_codes, k_scale,
                      static_cast<cudaStream_t>(stream));
}

int tara_set_kernel_events(void* start, void* stop) {
  if ((start == nullptr) != (stop == nullptr)) return TARA_ERR_NULL;
  t_ev_start = static_cast<cudaEvent_t>(start);
  t_ev_stop = static_cast<cudaEvent_t>(stop);
  return TARA_OK;
}

int tara_prepare_target_mask(const float* mask, int32_t F_in, int32_t Hp, int32_t Wp,
                             int32_t shot_len, int32_t frames_per_latent, int32_t F_lat,
                             int32_t Hq, int32_t Wq, float* m_out, void* stream_) {
  if (!mask || !m_out) return TARA_ERR_NULL;
  if (F_in < 1 || Hp < 1 || Wp < 1 || frames_per_latent < 1 || F_lat < 1 || Hq < 1 || Wq < 1)
    return TARA_ERR_SHAPE;
  if (shot_len < 5 || (shot_len - 5) % 17 != 0) return TARA_ERR_MASK_LENGTH;
  if (F_in != 1 && F_in != shot_len) return TARA_ERR_MASK_LENGTH;
  if (F_in > 1 && (long long)(F_lat - 1) * frames_per_latent >= shot_len) return TARA_ERR_SHAPE;
  if (F_lat > 65535 || Wq > 12288) return TARA_ERR_TOO_LARGE;   // Wq floats of shared memory
  if ((reinterpret_cast<uintptr_t>(mask) & 3u) != 0 || (reinterpret_cast<uintptr_t>(m_out) & 3u) != 0)
    return TARA_ERR_ALIGN;
  dim3 grid((unsigned)Hq, (unsigned)(F_in > 1 ? F_lat : 1));
  const bool narrow = Wp <= 8 * kMaskNarrowThreads && Wp % 4 == 0 &&
                      (reinterpret_cast<uintptr_t>(mask) & 15u) == 0;
  if (narrow)
    target_mask_narrow_kernel<<<grid, kMaskNarrowThreads, (size_t)Wq * sizeof(float),
                                static_cast<cudaStream_t>(stream_)>>>(
        mask, F_in, Hp, Wp, shot_len, frames_per_latent, F_lat, Hq, Wq, m_out);
  else
    target_mask_kernel<<<grid, kMaskThreads, (size_t)Wq * sizeof(float),
                         static_cast<cudaStream_t>(stream_)>>>(
        mask, F_in, Hp, Wp, shot_len, frames_per_latent, F_lat, Hq, Wq, m_out);
  return cudaGetLastError() == cudaSuccess ? TARA_OK : TARA_ERR_CUDA;
}

int tara_selftest_wait(int limit_us, int arrive, void* stream_) {
  if (limit_us < 1 || limit_us > 10000000) return TARA_ERR_PARAM;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  int rc = device_state(0, &st);
  if (rc != TARA_OK) return rc;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream_)>>>(
      st->status, (uint64_t)limit_us * 1000ull, arrive ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? TARA_OK : TARA_ERR_CUDA;
}

int tara_device_status(void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TARA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return TARA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return TARA_ERR_CUDA;
    // bit 1: a device-side check of the debug build failed; bit 0: a bounded wait gave up
    return (v & 2) ? TARA_ERR_DEBUG_CHECK : TARA_ERR_DEVICE_TIMEOUT;
  }
  return TARA_OK;
}

}  // extern "C"

extern "C" int tara_debug_build(void) {
#if defined(TARA_DEBUG) && TARA_DEBUG
  return 1;
#else
  return 0;
#endif
}

// ---------------------------------------------------------------------------------------
// Allocation-free variant of the 16-bit forward pass.
//
// Some callers may not allocate device memory at call time: code that runs under a
// framework's own memory pool (cudaMalloc there either fails, bypasses the pool's accounting,
// or synchronises the device in the middle of a step), and latency-bound serving loops that
// must never hit the driver's allocator.  For them the
// scratch the tensor-core path needs (tile summaries and per-key bias records) lives in a
// fixed device array that is part of the loaded module instead of the cached cudaMalloc
// workspace used by tara_attn_forward.
// ---------------------------------------------------------------------------------------
namespace tara {
namespace {

constexpr size_t kStaticScratchBytes = TARA_NOALLOC_SCRATCH_BYTES;

// Lives as long as the library is loaded, on every device that loads it.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

struct StaticState {
  bool ready = false;
  void* scratch = nullptr;   // device address of g_static_scratch on this device
  int* status = nullptr;     // device address of g_device_status on this device
};
std::mutex g_static_mu;
StaticState g_static[kMaxDevices];

// One-time set-up per device (the device must be current): device addresses of the two
// module variables.  The host-side names of __device__ variables are stand-ins that a kernel
// must never receive directly.
int static_state(StaticState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TARA_ERR_CUDA;
  StaticState& st = g_static[dev];
  if (!st.ready) {
    void* scratch = nullptr;
    void* status = nullptr;
    if (cudaGetSymbolAddress(&scratch, g_static_scratch) != cudaSuccess || scratch == nullptr)
      return TARA_ERR_CUDA;
    if (cudaGetSymbolAddress(&status, g_device_status) != cudaSuccess || status == nullptr)
      return TARA_ERR_CUDA;
    st.scratch = scratch;
    st.status = static_cast<int*>(status);
    st.ready = true;
  }
  *out = &st;
  return TARA_OK;
}

template <bool kBF16, int D>
int launch_tc_static(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const TcArgs& a, int B, int H, int ntiles, cudaStream_t stream) {
  constexpr int smem = TcShape<D>::kSmemBytes;
  if (tc_register_check(attn_tc_kernel<kBF16, D>) != TARA_OK) return TARA_ERR_CUDA;
  if (cudaFuncSetAttribute(attn_tc_kernel<kBF16, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return TARA_ERR_CUDA;
  dim3 grid((unsigned)((ntiles + 1) / 2), (unsigned)H, (unsigned)B);
  // a kernel-event pair armed by tara_set_kernel_events times this launch, as in
  // tara_attn_forward
  if (record_start(stream) != TARA_OK) return TARA_ERR_CUDA;
  attn_tc_kernel<kBF16, D><<<grid, kTcThreads, smem, stream>>>(mq, mk, mv, a);
  if (cudaGetLastError() != cudaSuccess) return TARA_ERR_CUDA;
  return record_stop(stream);
}

}  // namespace
}  // namespace tara

extern "C" int tara_attn_forward_noalloc(const tara_tensor* Q, const tara_tensor* K,
                                         const tara_tensor* V, const tara_token_meta* meta,
                                         const tara_params* p, tara_tensor* O, float* LSE,
                                         void* stream_) {
  using namespace tara;
  int rc = validate(Q, K, V, meta, p, O, LSE);
  if (rc != TARA_OK) return rc;
  if (Q->dtype == TARA_FP32) return TARA_ERR_DTYPE;   // the fp32 kernel needs no scratch
  if (p->qk_int8) return TARA_ERR_PARAM;              // 8-bit Q/K copies do not fit the scratch
  const int B = Q->B, H = Q->H, N = Q->N, D = Q->D;
  const int ntiles = (N + kTile - 1) / kTile;
  const size_t nsets = meta->batch_stride != 0 ? (size_t)B : 1;
  // the ascending and the descending copy of every record (tile_summary.cuh)
  const size_t rec_bytes = round_up(2 * nsets * (size_t)ntiles * sizeof(TileRec), 256);
  const size_t key_bytes = round_up(2 * nsets * (size_t)ntiles * kTile * sizeof(float4), 256);
  if (rec_bytes + key_bytes > kStaticScratchBytes) return TARA_ERR_TOO_LARGE;

  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const BiasParams bp = make_bias_params(p, D);
  std::lock_guard<std::mutex> lock(g_static_mu);
  StaticState* st = nullptr;
  if ((rc = static_state(&st)) != TARA_OK) return rc;
  if ((rc = get_encode_fn()) != TARA_OK) return rc;
  TileRec* recs = static_cast<TileRec*>(st->scratch);
  float4* keyinfo = reinterpret_cast<float4*>(static_cast<char*>(st->scratch) + rec_bytes);

  CUtensorMap mq, mk, mv;
  if (encode_qkv_map(&mq, Q) != TARA_OK || encode_qkv_map(&mk, K) != TARA_OK ||
      encode_qkv_map(&mv, V) != TARA_OK)
    return TARA_ERR_CUDA;
  // every record the attention kernel reads is rewritten here first, so the scratch needs no
  // clearing between calls
  tile_summary_kernel<<<dim3((unsigned)ntiles, (unsigned)nsets), 128, 0, stream>>>(
      meta->seg, meta->time_s, meta->pic, N, (long long)meta->batch_stride, ntiles, bp, recs,
      keyinfo, st->status);
  if (cudaGetLastError() != cudaSuccess) return TARA_ERR_CUDA;

  const TcArgs a =
      make_tc_args(meta, O, LSE, recs, keyinfo, N, H, ntiles, st->status, bp, nullptr, nullptr);
  const bool bf16 = Q->dtype == TARA_BF16;
  if (D == 128)
    return bf16 ? launch_pair<true>(Q, K, V, a, B, H, ntiles, stream, nullptr)
                : launch_pair<false>(Q, K, V, a, B, H, ntiles, stream, nullptr);
  return bf16 ? launch_tc_static<true, 64>(mq, mk, mv, a, B, H, ntiles, stream)
              : launch_tc_static<false, 64>(mq, mk, mv, a, B, H, ntiles, stream);
}
