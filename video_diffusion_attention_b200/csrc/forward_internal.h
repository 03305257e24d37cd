// forward_internal.h -- library-internal entry points shared by the C ABI and the host-buffer
// pipeline (not exported through include/tara_attn.h).
#pragma once

#include <cstddef>

#include "tara_attn.h"

namespace tara {

// Device workspace one tara_attn_forward call of this shape needs: the tile and per-key records
// of every metadata set and, with qk_int8, the 8-bit copies of Q and K and their scales.  0 for
// fp32 tensors (the CUDA-core kernel reads the metadata directly).
size_t forward_workspace_bytes(const tara_tensor* Q, const tara_token_meta* meta,
                               const tara_params* p);

// tara_attn_forward on a device workspace the caller owns (16-byte aligned, at least
// forward_workspace_bytes() long; TARA_ERR_TOO_LARGE if shorter).  No ordering against other
// calls is added: the caller must not let two calls that share `ws` overlap on the GPU, and
// calls with different workspaces on different streams may run concurrently.  plane_base: the
// index of this call's first (branch, head) plane within the larger call it was cut from; it
// fixes the order in which each plane's keys are walked, so that a plane's result is bit for
// bit the one the uncut call gives (0 for an uncut call; TARA_ERR_SHAPE if negative).
int forward_with_workspace(const tara_tensor* Q, const tara_tensor* K, const tara_tensor* V,
                           const tara_token_meta* meta, const tara_params* p, tara_tensor* O,
                           float* LSE, void* ws, size_t ws_bytes, void* stream,
                           long long plane_base);

}  // namespace tara
