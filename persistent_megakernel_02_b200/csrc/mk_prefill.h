// mk_prefill.h -- host interface of the batched prefill (mk_prefill.cu) used by
// the C ABI (mk_api.cu).
//
// A language model runs its prompt once and then decodes token by token; the two
// have different shapes ("One Megakernel is Not Enough: Predicting Where to Cut
// for Streaming Inference", section "Why where to cut matters more than whether
// to fuse").  Prefill is GEMM-shaped -- a tile of prompt tokens times a tile of
// weight rows -- so it runs on the tcgen05 tensor cores: per layer RMSNorm, the
// QKV GEMM (RoPE and the K/V cache writes fused in its epilogue), causal
// attention over the paged cache, the O GEMM (+ residual), RMSNorm, the gate/up
// GEMM (SwiGLU fused), the down GEMM (+ residual).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mk.h"
#include "mk_plan.h"

namespace mk {

struct PrefillPlan;

// Everything one batched prefill call needs from the handle.
struct PrefillCtx {
  const Dims* D;
  uint16_t* kv;            // KV cache [layer][physical page][kv head][K, V][PL][d]
  const int* page_table;   // [max_batch][pages_per_seq] (device)
  const float2* rope;      // [max_seq][d/2] (cos, sin) (device)
  uint32_t* err_code;      // the handle's device error word (first field)
  unsigned long long wait_limit_ns;
};

// True when the shape's GEMM tiles divide it (hidden, n_heads*head_dim and
// n_kv_heads*head_dim multiples of 128, ffn a multiple of 64).
bool prefill_supported(const Dims& D);

// Encodes the weight tensor maps and allocates the chunk workspace (at most
// `chunk` tokens per pass).  Returns MK_ERR_UNSUPPORTED for shapes outside
// prefill_supported.
mk_status prefill_create(const Dims& D, const mk_weights* w, int chunk, PrefillPlan** out);
void prefill_destroy(PrefillPlan* p);

// Runs the decoder layers over tokens_dev[0..n) (device int32) of slot `slot` at
// positions pos0 .. pos0 + n - 1: their K and V rows of every layer are written
// into the cache (the layers' remaining work is skipped where nothing reads it).
// Asynchronous on `st`; the cache must hold positions 0 .. pos0 - 1.
mk_status prefill_run(PrefillPlan* p, const PrefillCtx& c, const int* tokens_dev, int n, int slot, int pos0,
                      cudaStream_t st);

}  // namespace mk
