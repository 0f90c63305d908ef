// mk_api.cu -- the C ABI (include/mk.h): handle creation, tapes upload, one
// cooperative launch of the persistent kernel per decode step, prefill as a
// sequence of steps, error reporting, and the host-only tape checker.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "mk_kernel.cuh"
#include "mk_plan.h"
#include "mk_prefill.h"

using namespace mk;

namespace mk {
// host-side handles of mk_decode_kernel<nbt, spec>, one translation unit each (mk_inst.cu)
#define MK_DECL(s) \
  const void* decode_kernel_s##s##_n1(); \
  const void* decode_kernel_s##s##_n2(); \
  const void* decode_kernel_s##s##_n4(); \
  const void* decode_kernel_s##s##_n8();
MK_DECL(0)
MK_DECL(1)
MK_DECL(2)
#undef MK_DECL
}  // namespace mk

struct mk_ctx {
  mk_config cfg{};
  Dims D{};
  int dev = 0, n_sm = 0, nbt = 1;
  int spec = 0;  // kernel specialisation (mk_kernel.cuh, Spec)
  // KParams::hints: every op reads its inputs directly (measured faster than waiting on
  // the hint counters, also for the O projection's long wait on attention).  The
  // fault-injection hook works through hint waits, so it turns all of them on.
  int hints = 0;
  unsigned long long wait_limit_ns = 1000000000ull;
  SmemLayout sm{};
  std::vector<Tape> tapes;  // index nb - 1
  struct DevTape {
    Instr* instrs = nullptr;
    uint32_t* sm_off = nullptr;
  };
  std::vector<DevTape> dtapes;
  // region cut (mk_options.region_cut): tapes hold the decoder layers only, and the
  // final norm + LM head + argmax runs as a second launch from lm_tapes
  int region_cut = 0;
  std::vector<Tape> lm_tapes;
  std::vector<DevTape> lm_dtapes;
  const uint16_t* embed = nullptr;
  float* acts = nullptr;  // two sets of per-layer activation blocks (see KParams)
  long long set_floats = 0, layer_floats = 0, acc_base = 0, acc_floats = 0;
  long long claim_off = 0;  // claim counters of the dynamic tails, after the accumulators
  long long lmkey_off = 0;  // the step's greedy keys, after the claim counters
  int dyn_percent = kDynPercent;
  int off_q = 0, off_kvn = 0, off_o = 0, off_x1 = 0, off_a = 0;
  unsigned long long steps_run = 0;  // decode steps launched (activation-set parity)
  float* part = nullptr;
  uint16_t* kv = nullptr;  // [layer][physical page][kv head][K, V][PL][d]
  int* page_table = nullptr;
  // the layer matrices in page order (pack_weights): every unit's page is one
  // contiguous 16 KiB block, so the producer moves it with a single bulk copy
  uint16_t *pk_qkv = nullptr, *pk_gu = nullptr, *pk_dn = nullptr;
  // tensor-core tiles (Dims::tc): gate/up per layer, LM head
  uint16_t *pk_gu_tc = nullptr, *pk_lm_tc = nullptr;
  uint32_t* counters = nullptr;
  int n_counters = 0;
  ErrWord* err = nullptr;
  float2* rope = nullptr;
  int* tok_stage = nullptr;
  int tok_stage_cap = 0;
  // Host-path I/O: one device block [ids int32[8] | error word], so a host step
  // reads both back with a single copy, and its pinned host mirror; tokens of a
  // host step go in through pinned staging.
  unsigned char* io_dev = nullptr;
  int* ids_scratch = nullptr;       // io_dev + 0
  unsigned char* io_host = nullptr; // pinned, kIoBytes
  int* tok_host = nullptr;          // pinned, int32[8]
  int* tok_dev = nullptr;           // device, int32[8]
  float* logits_scratch = nullptr;
  unsigned long long step = 0;
  long long* prof = nullptr;
  int prof_stride = 0;
  // batched prefill on the tensor cores (mk_prefill.cu); null: prompts run token by
  // token through the decode kernel
  PrefillPlan* pf = nullptr;
  std::vector<void*> allocs;
};

// Prompts of at least this many tokens take the batched prefill (the rest run
// token by token through the decode kernel).
constexpr int kPrefillBatchMin = 16;
// tokens per batched-prefill pass (bounds its workspace)
constexpr int kPrefillChunk = 2048;
constexpr int kIoErrOff = 32;  // the error word's offset in the I/O block (after 8 ids)
constexpr int kIoBytes = kIoErrOff + (int)sizeof(ErrWord);

static const char* kVersion = "mk 0.1 (sm_100a persistent decode megakernel)";

extern "C" const char* mk_version(void) { return kVersion; }

namespace {

mk_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MK_OK;
  if (e == cudaErrorMemoryAllocation) return MK_ERR_OOM;
  return MK_ERR_CUDA;
}

#define MK_TRY(expr)                               \
  do {                                             \
    mk_status _s = (expr);                         \
    if (_s != MK_OK) return _s;                    \
  } while (0)

// Both activation sets to their empty state: float blocks hold the sentinel
// (0xFFFFFFFF), accumulators zero.
mk_status reset_acts(mk_ctx* h) {
  for (int set = 0; set < 2; ++set) {
    float* base = h->acts + (size_t)set * h->set_floats;
    MK_TRY(from_cuda(cudaMemset(base, 0xFF, sizeof(float) * h->acc_base)));
    MK_TRY(from_cuda(cudaMemset(base + h->acc_base, 0, sizeof(float) * (h->set_floats - h->acc_base))));
  }
  return MK_OK;
}

template <class T>
mk_status dalloc(mk_ctx* h, T** p, size_t count) {
  void* v = nullptr;
  size_t bytes = count * sizeof(T);
  if (bytes == 0) bytes = 16;
  cudaError_t e = cudaMalloc(&v, bytes);
  if (e != cudaSuccess) return from_cuda(e);
  h->allocs.push_back(v);
  cudaError_t z = cudaMemset(v, 0, bytes);
  if (z != cudaSuccess) return from_cuda(z);
  *p = static_cast<T*>(v);
  return MK_OK;
}

// Kernel specialisation of a shape (mk_kernel.cuh, Spec): 1 and 2 when every unit
// has the same row count and the attention one known form, else 0.
int kernel_spec(const Dims& D) {
  const int rq = 2 * D.RP, ro = D.Ro, rg = 2 * D.Rgu, rd = D.Rdn, rl = D.Rlm;
  if (rq == 4 && ro == 4 && rg == 4 && rd == 4 && rl == 4 && D.d == 64 && D.rep == 4 && !D.kv_fp16) return 1;
  if (rq == 2 && ro == 2 && rg == 2 && rd == 2 && rl == 2 && D.d == 128 && D.rep == 4 && D.kv_fp16) return 2;
  return 0;
}

// Whether the 8-lane kernel can run gate/up and the LM head on the tensor cores:
// the specialised Llama-3.2-1B-shaped kernel, whose staged activation (8 lanes x
// hidden fp32) has room for the MMA operand (16 rows of bf16 high/low parts x hidden).
bool tc_units(const Dims& D) {
  return kernel_spec(D) == 1 && lanes_template(D.max_batch) == 8 && D.H % 64 == 0 && D.F % 64 == 0 &&
         D.H >= 64 && D.H <= 2048;
}

// Tensor-core units of the 8-lane kernel by default (mk_options.tensor_core_units 0):
// the engine each op measured faster on with 8 lanes (bit 0 LM head, bit 1 gate/up).
// Llama-3.2-1B shape, batch 8, one box: CUDA cores 1504.3 us/step, LM head on tcgen05
// 1441.3, gate/up 1463.7, both 1387.6 (eight accumulators per unit, and the gate/up
// blocks kept out of the scheduler's cumulative balance).
constexpr int kTcDefault = 3;

std::string dims_from_config(const mk_config* c, int n_sm, Dims* D, int tc_sel = 0) {
  if (!(c->rms_eps >= 0.f) || !std::isfinite(c->rms_eps)) return "rms_eps must be finite and >= 0";
  if (!(c->rope_theta > 0.f)) return "rope_theta must be positive";
  if (c->rope_scaling) {
    if (!(c->rope_factor > 0.f) || !(c->rope_low_freq > 0.f) || !(c->rope_high_freq > c->rope_low_freq) ||
        c->rope_orig_max <= 0)
      return "invalid Llama-3 rope scaling parameters";
  }
  if (c->kv_dtype != 0 && c->kv_dtype != 1) return "kv_dtype must be 0 (bf16) or 1 (fp16)";
  std::string why = derive_dims(c->n_layers, c->hidden, c->n_heads, c->n_kv_heads, c->head_dim, c->ffn,
                                c->vocab, c->tied, c->rms_eps, c->max_batch, c->max_seq, n_sm, D);
  D->kv_fp16 = c->kv_dtype;
  if (why.empty()) D->tc = tc_units(*D) ? (tc_sel == 0 ? kTcDefault : tc_sel - 1) : 0;
  return why;
}

// Inverse frequencies theta^(-2i/d), i < d/2, with the optional Llama-3 rescaling:
// wavelengths 2 pi / f shorter than orig/high_freq are kept, longer than
// orig/low_freq divided by the factor, and in between blended linearly in
// orig/wavelength, f' = (1 - s) f / factor + s f with s = (orig/wl - low)/(high - low).
std::vector<double> inv_freq(const mk_config* c) {
  const int half = c->head_dim / 2;
  std::vector<double> f(half);
  const double pi = 3.14159265358979323846;
  for (int i = 0; i < half; ++i) {
    double base = std::pow((double)c->rope_theta, -2.0 * i / c->head_dim);
    if (c->rope_scaling) {
      const double lo = c->rope_low_freq, hi = c->rope_high_freq, orig = c->rope_orig_max;
      const double wl = 2.0 * pi / base;
      if (wl > orig / lo) {
        base = base / c->rope_factor;
      } else if (wl >= orig / hi) {
        const double t = (orig / wl - lo) / (hi - lo);
        base = (1.0 - t) * base / c->rope_factor + t * base;
      }
    }
    f[i] = base;
  }
  return f;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

mk_status check_weights(const mk_config* c, const mk_weights* w) {
  if (!w->embed || !w->final_norm) return MK_ERR_INVALID_ARG;
  if (c->tied ? (w->lm_head != nullptr) : (w->lm_head == nullptr)) return MK_ERR_INVALID_ARG;
  if (!aligned16(w->embed) || !aligned16(w->final_norm) || (w->lm_head && !aligned16(w->lm_head)))
    return MK_ERR_INVALID_ARG;
  const void* const* arrs[] = {w->attn_norm, w->wq, w->wk, w->wv, w->wo,
                               w->mlp_norm, w->w_gate, w->w_up, w->w_down};
  for (auto a : arrs) {
    if (!a) return MK_ERR_INVALID_ARG;
    for (int l = 0; l < c->n_layers; ++l)
      if (!a[l] || !aligned16(a[l])) return MK_ERR_INVALID_ARG;
  }
  return MK_OK;
}

// Packed-layer sizes (elements per layer).
size_t pk_gu_tc_elems(const Dims& D) { return (size_t)D.n_gu_tc * D.nkt * 128 * 64; }
size_t pk_qkv_elems(const Dims& D) { return (size_t)D.n_qkv * 2 * D.RP * D.H; }
size_t pk_gu_elems(const Dims& D) { return (size_t)D.n_gu * 2 * D.Rgu * D.H; }
size_t pk_dn_elems(const Dims& D) { return (size_t)D.n_ks * D.H * D.KS; }

// Copies row r (row_u4 16-byte words) from src[r], or zeros where src[r] is null,
// to dst + r * row_u4.
__global__ void pack_rows_kernel(const uint4* const* src, uint4* dst, long long n_rows, int row_u4) {
  const long long n = n_rows * row_u4;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / row_u4;
    const uint4* s = src[r];
    dst[e] = s ? s[e - r * row_u4] : make_uint4(0u, 0u, 0u, 0u);
  }
}

// Tensor-core tiles: block u, K tile kt is 128 rows x 64 bf16, row r's 16-byte
// chunk c stored at chunk (c ^ (r & 7)) of its 128-byte row (the 128-byte swizzle
// the MMA's shared-memory descriptor reads), tiles one after another in (u, kt)
// order, so the kernel streams every 16 KiB tile with one bulk copy.  Row r of
// block u comes from src[u * 128 + r] (zeros where null); rows are nkt * 64 long.
__global__ void pack_tc_tiles_kernel(const uint4* const* src, uint4* dst, long long n_rows, int nkt) {
  const long long n = n_rows * nkt * 8;  // 16-byte chunks
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(e & 7);
    const long long rest = e >> 3;
    const int r = (int)(rest & 127);
    const long long ut = rest >> 7;  // u * nkt + kt
    const int kt = (int)(ut % nkt);
    const long long u = ut / nkt;
    const uint4* s = src[u * 128 + r];
    dst[(ut * 128 + r) * 8 + (c ^ (r & 7))] = s ? s[(size_t)kt * 8 + c] : make_uint4(0u, 0u, 0u, 0u);
  }
}

mk_status pack_tc_tiles(const std::vector<const void*>& rows, void* dst, int nkt) {
  const uint4** d_src = nullptr;
  MK_TRY(from_cuda(cudaMalloc(&d_src, rows.size() * sizeof(void*))));
  cudaError_t e = cudaMemcpy(d_src, rows.data(), rows.size() * sizeof(void*), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) {
    pack_tc_tiles_kernel<<<1184, 256>>>(d_src, static_cast<uint4*>(dst), (long long)rows.size(), nkt);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  cudaFree(d_src);
  return from_cuda(e);
}

mk_status pack_rows(const std::vector<const void*>& rows, void* dst, int row_bytes) {
  const uint4** d_src = nullptr;
  MK_TRY(from_cuda(cudaMalloc(&d_src, rows.size() * sizeof(void*))));
  cudaError_t e = cudaMemcpy(d_src, rows.data(), rows.size() * sizeof(void*), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) {
    pack_rows_kernel<<<1184, 256>>>(d_src, static_cast<uint4*>(dst), (long long)rows.size(), row_bytes / 16);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  cudaFree(d_src);
  return from_cuda(e);
}

// Lay the layer matrices out in the order the producer streams them, one unit
// after another, each unit one contiguous page:
//   QKV   unit u: the RP rows of its RoPE first halves, then the RP second halves
//   GU    unit u: Rgu rows of W_gate, then the same Rgu rows of W_up (rows past
//         ffn in a ragged last unit are zero)
//   DOWN  K slice ks, rows r: W_down[r][ks*KS .. ks*KS + KS), slices one after
//         another, so the Rdn rows of a unit are adjacent
// A page made of several strided pieces streamed measurably slower than one
// contiguous block (Llama-3.2-1B batch 1: 538 vs 463 us per step).
mk_status pack_weights(mk_ctx* h, const mk_weights* w) {
  const Dims& D = h->D;
  const int half = D.d / 2;
  MK_TRY(dalloc(h, &h->pk_qkv, pk_qkv_elems(D) * D.L));
  MK_TRY(dalloc(h, &h->pk_gu, pk_gu_elems(D) * D.L));
  MK_TRY(dalloc(h, &h->pk_dn, pk_dn_elems(D) * D.L));
  const size_t rowH = (size_t)D.H;
  std::vector<const void*> rows;
  for (int l = 0; l < D.L; ++l)
    for (int u = 0; u < D.n_qkv; ++u) {
      const int P0 = u * D.RP, hg = P0 / half, i0 = P0 % half;
      const int sec = hg < D.Hq ? 0 : (hg < D.Hq + D.Hkv ? 1 : 2);
      const int hh = sec == 0 ? hg : (sec == 1 ? hg - D.Hq : hg - D.Hq - D.Hkv);
      const uint16_t* m = static_cast<const uint16_t*>(sec == 0 ? w->wq[l] : sec == 1 ? w->wk[l] : w->wv[l]);
      for (int hf = 0; hf < 2; ++hf)
        for (int j = 0; j < D.RP; ++j) rows.push_back(m + ((size_t)hh * D.d + i0 + hf * half + j) * rowH);
    }
  MK_TRY(pack_rows(rows, h->pk_qkv, D.H * 2));
  rows.clear();
  for (int l = 0; l < D.L; ++l)
    for (int u = 0; u < D.n_gu; ++u)
      for (int m = 0; m < 2; ++m)
        for (int j = 0; j < D.Rgu; ++j) {
          const int r = u * D.Rgu + j;
          const uint16_t* src = static_cast<const uint16_t*>(m == 0 ? w->w_gate[l] : w->w_up[l]);
          rows.push_back(r < D.F ? src + (size_t)r * rowH : nullptr);
        }
  MK_TRY(pack_rows(rows, h->pk_gu, D.H * 2));
  rows.clear();
  for (int l = 0; l < D.L; ++l)
    for (int ks = 0; ks < D.n_ks; ++ks)
      for (int r = 0; r < D.H; ++r)
        rows.push_back(static_cast<const uint16_t*>(w->w_down[l]) + (size_t)r * D.F + (size_t)ks * D.KS);
  MK_TRY(pack_rows(rows, h->pk_dn, D.KS * 2));
  if (D.tc & 2) {  // tensor-core tiles of gate/up, gate and up rows interleaved
    MK_TRY(dalloc(h, &h->pk_gu_tc, pk_gu_tc_elems(D) * D.L));
    rows.clear();
    for (int l = 0; l < D.L; ++l)
      for (int u = 0; u < D.n_gu_tc; ++u)
        for (int r = 0; r < 128; ++r) {
          const uint16_t* m = static_cast<const uint16_t*>((r & 1) ? w->w_up[l] : w->w_gate[l]);
          rows.push_back(m + (size_t)(64 * u + (r >> 1)) * rowH);
        }
    MK_TRY(pack_tc_tiles(rows, h->pk_gu_tc, D.nkt));
  }
  if (D.tc & 1) {  // tensor-core tiles of the LM head (rows past the vocabulary zero)
    MK_TRY(dalloc(h, &h->pk_lm_tc, (size_t)D.n_lm_tc * D.nkt * 128 * 64));
    rows.clear();
    const uint16_t* lm = static_cast<const uint16_t*>(D.tied ? w->embed : w->lm_head);
    for (int v = 0; v < D.n_lm_tc * 128; ++v) rows.push_back(v < D.V ? lm + (size_t)v * rowH : nullptr);
    MK_TRY(pack_tc_tiles(rows, h->pk_lm_tc, D.nkt));
  }
  return MK_OK;
}

// Resolve the device pointers each instruction streams from (see Instr::ptr).
void resolve_pointers(Tape& t, const Dims& D, const mk_weights* w, const mk_ctx* h) {
  const void* lm = D.tied ? w->embed : w->lm_head;
  for (Instr& I : t.instrs) {
    const int l = I.layer;
    I.ptr[0] = I.ptr[1] = I.ptr[2] = I.ptr[3] = nullptr;
    switch (I.op) {
      case OP_QKV: I.ptr[0] = h->pk_qkv + pk_qkv_elems(D) * l; I.ptr[3] = w->attn_norm[l]; break;
      case OP_O: I.ptr[0] = w->wo[l]; break;
      case OP_GU: I.ptr[0] = h->pk_gu + pk_gu_elems(D) * l; I.ptr[3] = w->mlp_norm[l]; break;
      case OP_DOWN: I.ptr[0] = h->pk_dn + pk_dn_elems(D) * l; break;
      case OP_LM: I.ptr[0] = lm; I.ptr[3] = w->final_norm; break;
      case OP_GU_TC: I.ptr[0] = h->pk_gu_tc + pk_gu_tc_elems(D) * l; I.ptr[3] = w->mlp_norm[l]; break;
      case OP_LM_TC: I.ptr[0] = h->pk_lm_tc; I.ptr[3] = w->final_norm; break;
      default: break;
    }
  }
}

// The kernel instantiations live in their own translation units (mk_inst.cu,
// compiled once per specialisation).
const void* kernel_for(int nbt, int spec) {
#define MK_PICK(s)                             \
  switch (nbt) {                               \
    case 1: return decode_kernel_s##s##_n1();  \
    case 2: return decode_kernel_s##s##_n2();  \
    case 4: return decode_kernel_s##s##_n4();  \
    default: return decode_kernel_s##s##_n8(); \
  }
  if (spec == 1) MK_PICK(1)
  if (spec == 2) MK_PICK(2)
  MK_PICK(0)
#undef MK_PICK
}

mk_status build(mk_ctx* h, const mk_weights* w, int want_pages) {
  const Dims& D = h->D;
  MK_TRY(pack_weights(h, w));
  // tapes, one per active batch size (two with the region cut: layers, LM head)
  auto upload = [&](Tape& t, std::vector<mk_ctx::DevTape>& dst) -> mk_status {
    resolve_pointers(t, D, w, h);
    mk_ctx::DevTape dt;
    MK_TRY(dalloc(h, &dt.instrs, t.instrs.size()));
    MK_TRY(dalloc(h, &dt.sm_off, t.sm_off.size()));
    MK_TRY(from_cuda(cudaMemcpy(dt.instrs, t.instrs.data(), t.instrs.size() * sizeof(Instr), cudaMemcpyHostToDevice)));
    MK_TRY(from_cuda(cudaMemcpy(dt.sm_off, t.sm_off.data(), t.sm_off.size() * 4, cudaMemcpyHostToDevice)));
    dst.push_back(dt);
    return MK_OK;
  };
  for (int nb = 1; nb <= D.max_batch; ++nb) {
    h->tapes.push_back(lower(D, h->n_sm, nb, h->dyn_percent, h->region_cut ? REGION_LAYERS : REGION_ALL));
    MK_TRY(upload(h->tapes.back(), h->dtapes));
    if (h->region_cut) {
      h->lm_tapes.push_back(lower(D, h->n_sm, nb, h->dyn_percent, REGION_LM));
      MK_TRY(upload(h->lm_tapes.back(), h->lm_dtapes));
    }
  }
  h->embed = (const uint16_t*)w->embed;
  // scratch and state
  const int S1 = h->tapes[0].S;  // nb = 1 has the most slices
  {
    const int MB = D.max_batch;
    long long off = 0;
    h->off_q = (int)off;   off += (long long)MB * D.qdim;
    h->off_kvn = (int)off; off += (long long)MB * 2 * D.kvdim;
    h->off_o = (int)off;   off += (long long)MB * D.qdim;
    h->off_x1 = (int)off;  off += (long long)MB * D.H;
    h->off_a = (int)off;   off += (long long)MB * D.F;
    h->layer_floats = (off + 7) / 8 * 8;
    h->acc_floats = 2LL * MB * D.H;  // 64-bit accumulators
    h->acc_base = h->layer_floats * D.L;
    h->claim_off = h->acc_base + h->acc_floats * D.L;
    h->lmkey_off = h->claim_off + (n_pools(D) + 3) / 4 * 4;
    h->set_floats = h->lmkey_off + 2 * kMaxNB;  // a whole number of 16-byte refill stores
    MK_TRY(dalloc(h, &h->acts, (size_t)2 * h->set_floats));
    MK_TRY(reset_acts(h));
  }
  MK_TRY(dalloc(h, &h->part, (size_t)kMaxNB * D.Hkv * S1 * D.rep * (D.d + 2)));
  const size_t kv = (size_t)D.L * D.n_phys_pages * D.Hkv * D.PL * D.d;
  MK_TRY(dalloc(h, &h->kv, 2 * kv));
  std::vector<int> pt((size_t)D.max_batch * D.pages_per_seq);
  for (size_t i = 0; i < pt.size(); ++i) pt[i] = (int)i;  // slot s owns pages s*pps .. s*pps+pps-1
  MK_TRY(dalloc(h, &h->page_table, pt.size()));
  MK_TRY(from_cuda(cudaMemcpy(h->page_table, pt.data(), pt.size() * 4, cudaMemcpyHostToDevice)));
  h->n_counters = n_counters(D);
  MK_TRY(dalloc(h, &h->counters, (size_t)2 * h->n_counters));
  MK_TRY(dalloc(h, &h->io_dev, (size_t)kIoBytes));
  h->ids_scratch = reinterpret_cast<int*>(h->io_dev);
  h->err = reinterpret_cast<ErrWord*>(h->io_dev + kIoErrOff);
  MK_TRY(dalloc(h, &h->tok_dev, kMaxNB));
  MK_TRY(from_cuda(cudaMallocHost(&h->io_host, kIoBytes)));
  MK_TRY(from_cuda(cudaMallocHost(&h->tok_host, sizeof(int) * kMaxNB)));
  // RoPE table: cos/sin of pos * inv_freq[i], computed in double
  const int half = D.d / 2;
  std::vector<double> f = inv_freq(&h->cfg);
  std::vector<float2> tab((size_t)D.max_seq * half);
  for (int p = 0; p < D.max_seq; ++p)
    for (int i = 0; i < half; ++i) {
      const double ang = (double)p * f[i];
      tab[(size_t)p * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
  MK_TRY(dalloc(h, &h->rope, tab.size()));
  MK_TRY(from_cuda(cudaMemcpy(h->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice)));
  // shared memory and kernel attributes
  int max_dyn = 0;
  MK_TRY(from_cuda(cudaDeviceGetAttribute(&max_dyn, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->dev)));
  h->sm = smem_layout(D, h->nbt, max_dyn, want_pages);
  if (h->sm.ring_pages < kConsumerWarps) return MK_ERR_UNSUPPORTED;
  if (h->sm.ring_pages > 64) return MK_ERR_UNSUPPORTED;
  h->spec = kernel_spec(D);
  for (int nbt : {1, 2, 4, 8})
    MK_TRY(from_cuda(cudaFuncSetAttribute(kernel_for(nbt, h->spec), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          h->sm.total)));
  int blocks = 0;
  MK_TRY(from_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kernel_for(8, h->spec), kThreads,
                                                                  h->sm.total)));
  if (blocks < 1) return MK_ERR_UNSUPPORTED;
  return from_cuda(cudaDeviceSynchronize());
}


// One launch of n_steps decode steps (see KParams for the token / ids / logits modes).
mk_status launch_step(mk_ctx* h, int nb, const int* tokens_dev, const int* pos, const int* slot,
                      float* logits, int* ids, cudaStream_t st, int n_steps = 1, int chain = 1,
                      int ids_stride = 0, int logits_last = 0, int region = REGION_ALL) {
  const Dims& D = h->D;
  const bool lm = region == REGION_LM;
  const Tape& t = lm ? h->lm_tapes[nb - 1] : h->tapes[nb - 1];
  const mk_ctx::DevTape& dt = lm ? h->lm_dtapes[nb - 1] : h->dtapes[nb - 1];
  KParams p{};
  p.instrs = dt.instrs;
  p.sm_off = dt.sm_off;
  p.S = t.S;
  p.embed = h->embed;
  p.acts = h->acts;
  p.set_floats = h->set_floats;
  p.layer_floats = h->layer_floats;
  p.off_q = h->off_q; p.off_kvn = h->off_kvn; p.off_o = h->off_o;
  p.off_x1 = h->off_x1; p.off_a = h->off_a;
  p.acc_base = h->acc_base;
  p.acc_floats = h->acc_floats;
  p.claim_off = h->claim_off;
  p.lmkey_off = h->lmkey_off;
  p.parity0 = (int)(h->steps_run & 1);
  p.hints = h->hints;
  p.part = h->part;
  p.kv = h->kv; p.page_table = h->page_table;
  const int par = (int)(h->step & 1);
  p.ctr = h->counters + (size_t)par * h->n_counters;
  p.ctr_next = h->counters + (size_t)(1 - par) * h->n_counters;
  p.n_counters = h->n_counters;
  p.err = h->err;
  p.rope = h->rope;
  p.nb = nb;
  p.n_steps = n_steps;
  p.chain = chain;
  p.ids_stride = ids_stride;
  p.logits_last = logits_last;
  p.tokens = tokens_dev;
  for (int b = 0; b < kMaxNB; ++b) {
    p.pos[b] = b < nb ? pos[b] : 0;
    p.slot[b] = b < nb ? slot[b] : 0;
  }
  p.logits = logits;
  p.ids = ids;
  p.wait_limit_ns = h->wait_limit_ns;
  p.prof = h->prof;
  p.prof_stride = h->prof_stride;
  p.ring_pages = h->sm.ring_pages;
  p.act_off = h->sm.ring_pages * kPageBytes;
  p.bar_off = h->sm.bar_off;
  p.misc_off = h->sm.misc_off;
  p.D = D;
  void* args[] = {&p};
  const int nbt = lanes_template(nb);
  cudaError_t e = cudaLaunchCooperativeKernel(kernel_for(nbt, h->spec), dim3(h->n_sm), dim3(kThreads), args,
                                              (size_t)h->sm.total, st);
  h->step++;
  // the layers launch of a cut step shares the LM launch's activation set
  if (e == cudaSuccess && region != REGION_LAYERS) h->steps_run += (unsigned long long)n_steps;
  return from_cuda(e);
}

// n_steps decode steps (the launch_step modes).  One launch, or with the region cut
// two per step: the layers, then the LM head.  Step t of a cut run reads its tokens
// where the single launch's step t would (the previous step's ids when chained),
// writes its ids and logits where that step would, at positions pos[b] + t.
mk_status run_steps(mk_ctx* h, int nb, const int* tokens_dev, const int* pos, const int* slot, float* logits,
                    int* ids, cudaStream_t st, int n_steps, int chain, int ids_stride, int logits_last) {
  if (!h->region_cut)
    return launch_step(h, nb, tokens_dev, pos, slot, logits, ids, st, n_steps, chain, ids_stride, logits_last);
  const size_t V = (size_t)h->D.V;
  for (int t = 0; t < n_steps; ++t) {
    const int* tok = (chain && t > 0) ? ids + (size_t)(t - 1) * ids_stride : tokens_dev + (size_t)(chain ? 0 : t) * nb;
    int pt[kMaxNB];
    for (int b = 0; b < nb; ++b) pt[b] = pos[b] + t;
    float* lg = logits_last ? (t == n_steps - 1 ? logits : nullptr) : (logits ? logits + (size_t)t * nb * V : nullptr);
    int* id = ids + (size_t)t * ids_stride;
    MK_TRY(launch_step(h, nb, tok, pt, slot, nullptr, id, st, 1, 0, 0, 0, REGION_LAYERS));
    MK_TRY(launch_step(h, nb, tok, pt, slot, lg, id, st, 1, 0, 0, 0, REGION_LM));
  }
  return MK_OK;
}

mk_status read_error(mk_ctx* h, ErrWord* out) {
  return from_cuda(cudaMemcpy(out, h->err, sizeof(ErrWord), cudaMemcpyDeviceToHost));
}

mk_status status_of(const ErrWord& e) {
  switch (e.code) {
    case 0: return e.abort ? MK_ERR_ABORTED : MK_OK;
    case E_BAD_TOKEN: return MK_ERR_DEVICE_FAULT;
    default: return MK_ERR_TIMEOUT;
  }
}

}  // namespace

extern "C" mk_status mk_rope_inv_freq(const mk_config* cfg, double* out, int32_t n) {
  if (!cfg || !out || cfg->head_dim < 2 || n < cfg->head_dim / 2) return MK_ERR_INVALID_ARG;
  if (!(cfg->rope_theta > 0.f)) return MK_ERR_INVALID_ARG;
  if (cfg->rope_scaling && (!(cfg->rope_factor > 0.f) || !(cfg->rope_low_freq > 0.f) ||
                            !(cfg->rope_high_freq > cfg->rope_low_freq) || cfg->rope_orig_max <= 0))
    return MK_ERR_INVALID_ARG;
  const std::vector<double> f = inv_freq(cfg);
  for (size_t i = 0; i < f.size(); ++i) out[i] = f[i];
  return MK_OK;
}

extern "C" mk_status mk_plan_check(const mk_config* cfg, int32_t n_sm, int32_t nb, int32_t fault,
                                   int32_t dyn_percent, int32_t region, int32_t tensor_core_units,
                                   mk_plan_report* rep) {
  if (!cfg || !rep || n_sm < 1 || dyn_percent < 0 || dyn_percent > 90) return MK_ERR_INVALID_ARG;
  if (region < REGION_ALL || region > REGION_LM) return MK_ERR_INVALID_ARG;
  if (tensor_core_units < 0 || tensor_core_units > 4) return MK_ERR_INVALID_ARG;
  memset(rep, 0, sizeof(*rep));
  Dims D;
  std::string why = dims_from_config(cfg, n_sm, &D, tensor_core_units);
  if (!why.empty()) return MK_ERR_UNSUPPORTED;
  if (nb < 1 || nb > D.max_batch) return MK_ERR_INVALID_ARG;
  Tape t = lower(D, n_sm, nb, dyn_percent > 0 ? dyn_percent : kDynPercent, region);
  if (fault == 3) {  // shrink the LM head's claim range by one unit on one SM
    for (auto& I : t.instrs)
      if (I.op == OP_LM && I.pool) { I.pool_u1 -= 1; break; }
  } else if (fault == 1) {  // drop one signal: the first QKV instruction of the last layer
    for (auto& I : t.instrs)
      if (I.op == OP_QKV && I.layer == D.L - 1) { I.sig = kNoCounter; break; }
  } else if (fault == 2) {  // raise one wait target
    for (auto& I : t.instrs)
      if (I.dep != kNoCounter) { I.dep_target += 1; break; }
  }
  SimReport r = simulate(D, n_sm, t);
  rep->n_instr_total = r.n_instr_total;
  rep->n_counters = t.n_counters;
  rep->max_instr_per_sm = r.max_instr_per_sm;
  rep->bytes_min_sm = r.bytes_min;
  rep->bytes_max_sm = r.bytes_max;
  rep->deadlock_free = r.deadlock_free;
  rep->coverage_ok = r.coverage_ok;
  rep->targets_ok = r.targets_ok;
  rep->attn_slices = t.S;
  SmemLayout s = smem_layout(D, lanes_template(D.max_batch), 232448, 0);
  rep->ring_pages = s.ring_pages;
  rep->smem_bytes = s.total;
  return MK_OK;
}

extern "C" mk_status mk_create(const mk_config* cfg, const mk_weights* w, const mk_options* opt,
                               mk_handle* out) {
  if (!cfg || !w || !out) return MK_ERR_INVALID_ARG;
  *out = nullptr;
  mk_options o{};
  if (opt) o = *opt;
  if (o.wait_limit_ms < 0 || o.n_sm < 0 || o.ring_pages < 0 || o.device < 0) return MK_ERR_INVALID_ARG;
  if (o.dyn_percent < 0 || o.dyn_percent > 90) return MK_ERR_INVALID_ARG;
  if (o.region_cut != 0 && o.region_cut != 1) return MK_ERR_INVALID_ARG;
  if (o.tensor_core_units < 0 || o.tensor_core_units > 4) return MK_ERR_INVALID_ARG;
  Dims D;
  std::string why = dims_from_config(cfg, 148, &D);  // validation only; rederived below
  if (!why.empty()) return MK_ERR_UNSUPPORTED;
  MK_TRY(check_weights(cfg, w));
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) return MK_ERR_CUDA;
  if (o.device >= ndev) return MK_ERR_INVALID_ARG;
  MK_TRY(from_cuda(cudaSetDevice(o.device)));
  int sms = 0, major = 0, coop = 0;
  MK_TRY(from_cuda(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, o.device)));
  MK_TRY(from_cuda(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, o.device)));
  MK_TRY(from_cuda(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, o.device)));
  if (major != 10 || !coop) return MK_ERR_UNSUPPORTED;
  mk_ctx* h = new mk_ctx();
  h->cfg = *cfg;
  h->dev = o.device;
  h->n_sm = o.n_sm > 0 ? std::min(o.n_sm, sms) : sms;
  h->wait_limit_ns = (unsigned long long)(o.wait_limit_ms > 0 ? o.wait_limit_ms : 1000) * 1000000ull;
  h->dyn_percent = o.dyn_percent > 0 ? o.dyn_percent : kDynPercent;
  h->region_cut = o.region_cut ? 1 : 0;
  why = dims_from_config(cfg, h->n_sm, &h->D, o.tensor_core_units);
  h->nbt = lanes_template(cfg->max_batch);
  mk_status s = why.empty() ? build(h, w, o.ring_pages) : MK_ERR_UNSUPPORTED;
  if (s == MK_OK && !o.prefill_tokenwise && prefill_supported(h->D))
    s = prefill_create(h->D, w, std::min(kPrefillChunk, h->D.max_seq), &h->pf);
  if (s == MK_OK && o.profile) {
    int stride = 1;
    for (const auto* ts : {&h->tapes, &h->lm_tapes})
      for (const Tape& t : *ts)
        for (int sm = 0; sm < h->n_sm; ++sm) stride = std::max(stride, (int)(t.sm_off[sm + 1] - t.sm_off[sm]));
    h->prof_stride = stride;
    s = dalloc(h, &h->prof, (size_t)h->n_sm * stride * kProfSlots);
  }
  if (s == MK_OK && o.debug_fault == 1) {
    h->hints = 0xFE;
    // test hook: one wait (the first layer-0 O projection of SM 0's tape for every
    // batch size) gets a target one above what its counter can reach
    for (size_t k = 0; k < h->tapes.size(); ++k) {
      Tape& t = h->tapes[k];
      for (uint32_t i = t.sm_off[0]; i < t.sm_off[1]; ++i)
        if (t.instrs[i].dep != kNoCounter) {
          t.instrs[i].dep_target += 1;
          s = from_cuda(cudaMemcpy(h->dtapes[k].instrs + i, &t.instrs[i], sizeof(Instr), cudaMemcpyHostToDevice));
          break;
        }
    }
  }
  if (s != MK_OK) {
    mk_destroy(h);
    return s;
  }
  *out = h;
  return MK_OK;
}

extern "C" mk_status mk_destroy(mk_handle h) {
  if (!h) return MK_ERR_INVALID_ARG;
  cudaSetDevice(h->dev);
  cudaDeviceSynchronize();
  for (void* p : h->allocs) cudaFree(p);
  prefill_destroy(h->pf);
  if (h->tok_stage) cudaFree(h->tok_stage);
  if (h->io_host) cudaFreeHost(h->io_host);
  if (h->tok_host) cudaFreeHost(h->tok_host);
  if (h->logits_scratch) cudaFree(h->logits_scratch);
  delete h;
  return MK_OK;
}

extern "C" mk_status mk_decode_step(mk_handle h, int32_t nb, const int32_t* tokens_dev,
                                    const int32_t* positions, float* logits_dev, int32_t* ids_dev,
                                    void* stream) {
  if (!h || !tokens_dev || !positions || !ids_dev) return MK_ERR_INVALID_ARG;
  if (nb < 1 || nb > h->D.max_batch) return MK_ERR_INVALID_ARG;
  int slot[kMaxNB];
  for (int b = 0; b < nb; ++b) {
    if (positions[b] < 0 || positions[b] >= h->D.max_seq) return MK_ERR_INVALID_ARG;
    slot[b] = b;
  }
  cudaSetDevice(h->dev);
  return run_steps(h, nb, tokens_dev, positions, slot, logits_dev, ids_dev, (cudaStream_t)stream, 1, 1, 0, 0);
}

extern "C" mk_status mk_decode_steps(mk_handle h, int32_t nb, int32_t n_steps, const int32_t* tokens_dev,
                                     const int32_t* positions, float* logits_dev, int32_t* ids_dev,
                                     void* stream) {
  if (!h || !tokens_dev || !positions || !ids_dev) return MK_ERR_INVALID_ARG;
  if (nb < 1 || nb > h->D.max_batch || n_steps < 1) return MK_ERR_INVALID_ARG;
  int slot[kMaxNB];
  for (int b = 0; b < nb; ++b) {
    if (positions[b] < 0 || (long long)positions[b] + n_steps > h->D.max_seq) return MK_ERR_INVALID_ARG;
    slot[b] = b;
  }
  cudaSetDevice(h->dev);
  return run_steps(h, nb, tokens_dev, positions, slot, logits_dev, ids_dev, (cudaStream_t)stream, n_steps,
                   /*chain=*/1, /*ids_stride=*/nb, /*logits_last=*/0);
}

extern "C" mk_status mk_sync(mk_handle h, void* stream) {
  if (!h) return MK_ERR_INVALID_ARG;
  cudaSetDevice(h->dev);
  MK_TRY(from_cuda(cudaStreamSynchronize((cudaStream_t)stream)));
  ErrWord e;
  MK_TRY(read_error(h, &e));
  return status_of(e);
}

extern "C" mk_status mk_decode_step_host(mk_handle h, int32_t nb, const int32_t* tokens_host,
                                         const int32_t* positions, float* logits_host,
                                         int32_t* ids_host, void* stream) {
  if (!h || !tokens_host || !positions || !ids_host) return MK_ERR_INVALID_ARG;
  if (nb < 1 || nb > h->D.max_batch) return MK_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  cudaSetDevice(h->dev);
  if (logits_host && !h->logits_scratch)
    MK_TRY(from_cuda(cudaMalloc(&h->logits_scratch, sizeof(float) * (size_t)kMaxNB * h->D.V)));
  // tokens in through pinned staging; the step; ids and the error word back in one
  // copy into pinned memory; one wait for the stream
  memcpy(h->tok_host, tokens_host, sizeof(int) * nb);
  MK_TRY(from_cuda(cudaMemcpyAsync(h->tok_dev, h->tok_host, sizeof(int) * nb, cudaMemcpyHostToDevice, st)));
  MK_TRY(mk_decode_step(h, nb, h->tok_dev, positions, logits_host ? h->logits_scratch : nullptr,
                        h->ids_scratch, stream));
  MK_TRY(from_cuda(cudaMemcpyAsync(h->io_host, h->io_dev, kIoBytes, cudaMemcpyDeviceToHost, st)));
  if (logits_host)
    MK_TRY(from_cuda(cudaMemcpyAsync(logits_host, h->logits_scratch, sizeof(float) * (size_t)nb * h->D.V,
                                     cudaMemcpyDeviceToHost, st)));
  MK_TRY(from_cuda(cudaStreamSynchronize(st)));
  memcpy(ids_host, h->io_host, sizeof(int) * nb);
  ErrWord e;
  memcpy(&e, h->io_host + kIoErrOff, sizeof e);
  return status_of(e);
}

extern "C" mk_status mk_prefill(mk_handle h, int32_t seq, const int32_t* tokens_host, int32_t n,
                                int32_t start_pos, float* logits_last_dev, int32_t* id_last_host,
                                void* stream) {
  if (!h || !tokens_host || n < 1) return MK_ERR_INVALID_ARG;
  if (seq < 0 || seq >= h->D.max_batch || start_pos < 0 || (long long)start_pos + n > h->D.max_seq)
    return MK_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (tokens_host[i] < 0 || tokens_host[i] >= h->D.V) return MK_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  cudaSetDevice(h->dev);
  if (h->tok_stage_cap < n) {
    MK_TRY(from_cuda(cudaStreamSynchronize(st)));
    if (h->tok_stage) cudaFree(h->tok_stage);
    h->tok_stage = nullptr;
    h->tok_stage_cap = 0;
    MK_TRY(from_cuda(cudaMalloc(&h->tok_stage, sizeof(int) * (size_t)std::max(n, kMaxNB))));
    h->tok_stage_cap = std::max(n, kMaxNB);
  }
  // pageable source: the copy completes before the call returns
  MK_TRY(from_cuda(cudaMemcpyAsync(h->tok_stage, tokens_host, sizeof(int) * n, cudaMemcpyHostToDevice, st)));
  MK_TRY(from_cuda(cudaStreamSynchronize(st)));
  int pos = start_pos, slot = seq;
  const int* first = h->tok_stage;
  if (h->pf && n - 1 >= kPrefillBatchMin) {
    // every token but the last through the batched layers (their K/V rows into the
    // cache); the last one through the decode kernel, which gives its logits and id
    PrefillCtx c;
    c.D = &h->D;
    c.kv = h->kv;
    c.page_table = h->page_table;
    c.rope = h->rope;
    c.err_code = &h->err->code;
    c.wait_limit_ns = h->wait_limit_ns;
    MK_TRY(prefill_run(h->pf, c, h->tok_stage, n - 1, seq, start_pos, st));
    pos = start_pos + n - 1;
    first = h->tok_stage + n - 1;
    n = 1;
  }
  // one launch runs the (rest of the) prompt: step i takes token i at position
  // pos + i; only the last step's logits are kept, every step overwrites the id
  MK_TRY(run_steps(h, 1, first, &pos, &slot, logits_last_dev, h->ids_scratch, st, n,
                   /*chain=*/0, /*ids_stride=*/0, /*logits_last=*/1));
  if (id_last_host) {
    MK_TRY(from_cuda(cudaMemcpyAsync(id_last_host, h->ids_scratch, sizeof(int), cudaMemcpyDeviceToHost, st)));
    return mk_sync(h, stream);
  }
  return MK_OK;
}

extern "C" mk_status mk_profile_read(mk_handle h, int64_t* out, int64_t cap, int32_t* n_sm,
                                     int32_t* stride) {
  if (!h || !n_sm || !stride) return MK_ERR_INVALID_ARG;
  *n_sm = h->n_sm;
  *stride = h->prof_stride;
  if (!h->prof) return MK_ERR_INVALID_ARG;
  const int64_t need = (int64_t)h->n_sm * h->prof_stride * kProfSlots;
  if (!out || cap < need) return MK_ERR_INVALID_ARG;
  cudaSetDevice(h->dev);
  MK_TRY(from_cuda(cudaDeviceSynchronize()));
  MK_TRY(from_cuda(cudaMemcpy(out, h->prof, need * sizeof(int64_t), cudaMemcpyDeviceToHost)));
  return from_cuda(cudaMemset(h->prof, 0, need * sizeof(int64_t)));  // accumulators restart
}

extern "C" mk_status mk_get_error(mk_handle h, char* buf, int32_t len) {
  if (!h) return MK_ERR_INVALID_ARG;
  cudaSetDevice(h->dev);
  MK_TRY(from_cuda(cudaDeviceSynchronize()));
  ErrWord e;
  MK_TRY(read_error(h, &e));
  if (buf && len > 0) {
    const char* what = "none";
    switch (e.code) {
      case E_WAIT_COUNTER: what = "counter wait timed out"; break;
      case E_WAIT_FULL: what = "ring page arrival wait timed out"; break;
      case E_WAIT_EMPTY: what = "ring page release wait timed out"; break;
      case E_BAD_TOKEN: what = "token out of range"; break;
      case E_DRAIN: what = "in-flight copy drain timed out"; break;
      case E_WAIT_DATA: what = "activation element wait timed out"; break;
      default: break;
    }
    snprintf(buf, (size_t)len, "%s (code %u, sm %u, instr %u, info %u, abort %u)", what, e.code, e.sm,
             e.instr, e.info, e.abort);
  }
  return status_of(e);
}

extern "C" mk_status mk_clear_error(mk_handle h) {
  if (!h) return MK_ERR_INVALID_ARG;
  cudaSetDevice(h->dev);
  MK_TRY(from_cuda(cudaDeviceSynchronize()));
  MK_TRY(from_cuda(cudaMemset(h->err, 0, sizeof(ErrWord))));
  MK_TRY(from_cuda(cudaMemset(h->counters, 0, sizeof(uint32_t) * 2 * h->n_counters)));
  // an aborted step may have left written elements behind: every set back to its empty state
  MK_TRY(reset_acts(h));
  return from_cuda(cudaDeviceSynchronize());
}
