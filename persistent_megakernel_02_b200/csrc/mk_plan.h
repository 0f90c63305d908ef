// mk_plan.h -- the instruction tape format shared by the host scheduler and the
// persistent kernel, plus the shape parameters both derive from a config.
//
// The per-SM "execution plan" of the Hazy megakernel article (section
// "Megakernel: a deep-fusion design from scratch"): an ordered list of fused
// instructions per SM whose dependencies are fixed before the run.  Here an
// instruction names an op, a layer, a contiguous range of work units (each unit
// is exactly one shared-memory page of weights, or one attention slice), the
// counter it waits on with its target, and the counter it bumps when done.
// Ranges keep the kernel free of per-unit table lookups: a unit id is u0 + k.
// The streaming phases end with a dynamic tail that SMs claim at run time.
#pragma once

#include <stdint.h>

#include <string>
#include <vector>

#if defined(__CUDACC__)
#define MK_HD __host__ __device__
#else
#define MK_HD
#endif

namespace mk {

enum Op : uint8_t {
  OP_QKV = 1,   // RMSNorm(x) -> rows of Wq|Wk|Wv -> RoPE -> q scratch / K,V cache
  OP_ATTN = 2,  // one slice of a (lane, kv head) over a range of KV pages -> partial; last merges
  OP_O = 3,     // rows of Wo . o -> x1 = residual + Wo . o
  OP_GU = 4,    // RMSNorm(x) -> rows of Wgate and Wup -> a = silu(g) * u
  OP_DOWN = 5,  // rows of Wdown over one K slice . a -> that slice's partial of the residual
  OP_LM = 6,    // RMSNorm(x) -> rows of the LM head -> logits, running argmax; last reduces
  // 8-lane kernels of handles with packed tensor-core tiles (Dims::tc): the same
  // ops on tcgen05, a unit being one 128-row block over the whole K (nkt pages of
  // 128 rows x 64 in the 128-byte swizzled layout)
  OP_GU_TC = 7,  // block u: rows 2i / 2i + 1 = W_gate / W_up row 64 u + i -> a = silu(g) * u
  OP_LM_TC = 8,  // block u: LM-head rows 128 u .. 128 u + 127 -> logits, running argmax
};

constexpr int kPageBytes = 16384;      // one ring page
constexpr int kMaxNB = 8;              // lanes (sequences) per step
constexpr int kConsumerWarps = 8;      // warps 1..8 compute; warp 0 loads the ring
constexpr int kThreads = 32 * (1 + kConsumerWarps);
constexpr int kActFloatsMax = 16384;   // max_batch * K of the staged activation
constexpr int kMaxKS = 8;              // down-projection K slices (the residual sums them)
constexpr int kProfSlots = 32;         // int64 fields of one profile record
constexpr uint16_t kNoCounter = 0xFFFF;

// counters of one layer
enum : int { C_QKV = 0, C_ATTN = 1, C_O = 2, C_GU = 3, C_DOWN = 4, kCountersPerLayer = 5 };

struct Instr {            // 64 bytes
  uint8_t op;
  uint8_t arg;            // OP_DOWN: K-slice index
  uint16_t layer;
  uint32_t u0;            // units of the instruction are u0 .. u0 + n_units - 1
  uint32_t n_units;
  uint16_t dep;           // counter waited on before the instruction (kNoCounter: none)
  uint16_t sig;           // counter incremented once when the instruction is done
  uint32_t dep_target;    // value `dep` must reach in this step
  // Dynamic tail (gate/up, down, LM head).  After its static units the SM claims
  // chunks of (pool >> 24) units from [pool_u0, pool_u1), a range shared by every
  // SM of the phase, through claim counter (pool & 0xFFFFFF) - 1 of the step's
  // activation set, until the range is exhausted.  pool == 0: static units only.
  uint32_t pool;
  uint32_t pool_u0, pool_u1;
  // device pointers resolved when the handle is created, so the kernel needs no
  // table lookup per instruction: [0] the weights the producer streams (QKV, GU,
  // DOWN: the layer's packed matrix, every unit one contiguous page; O: Wo; LM:
  // the head), [1..2] unused, [3] the bf16 RMSNorm gain the consumers stage with
  // (QKV, GU, LM)
  const void* ptr[4];
};
static_assert(sizeof(Instr) == 64, "Instr layout");

// Shape parameters of one handle (identical for every tape of the handle).
struct Dims {
  int L, H, Hq, Hkv, d, F, V, qdim, kvdim, rep;
  int RP;         // QKV: half-split pairs per unit (unit rows = 2*RP)
  int Ro, Rgu, Rdn, Rlm;  // rows per unit of O, gate/up (each), down, LM head
  int n_ks, KS;   // down projection: K slices and their width
  int PL;         // positions per KV page
  int pages_per_seq;
  int n_phys_pages;   // KV pages per layer per kv head (all slots)
  int max_batch, max_seq;
  int n_qkv, n_o, n_gu, n_dn, n_lm;   // units per op per layer (n_dn per K slice)
  float eps;
  int tied;
  int kv_fp16;    // KV cache element: 0 bf16, 1 fp16
  // tensor-core units in the 8-lane tapes: bit 0 the LM head, bit 1 gate/up (0: none)
  int tc;
  int nkt;        // 64-wide K tiles of a hidden-size row (tc units)
  int n_gu_tc, n_lm_tc;  // 128-row blocks of gate/up (F / 64) and of the LM head
};

// Which part of a decode step a tape holds.  The whole step is one launch; the
// region cut splits it into two launches, the decoder layers and then the final
// norm + LM head + argmax ("One Megakernel is Not Enough: Predicting Where to Cut
// for Streaming Inference", section "Four observations": two megakernels can beat
// one for a language model).  The LM-head tape waits on no counter: the launch
// boundary orders it after the layers.
enum Region : int { REGION_ALL = 0, REGION_LAYERS = 1, REGION_LM = 2 };

// One tape: the instruction lists of every SM for one active batch size.
struct Tape {
  int nb = 0;
  int region = REGION_ALL;
  int tc = 0;                     // gate/up and LM head as tensor-core units
  int S = 1;                      // attention slices per (lane, kv head)
  int n_counters = 0;
  std::vector<uint32_t> sm_off;   // n_sm + 1 offsets into instrs
  std::vector<Instr> instrs;
};

// Share of the gate/up, down and LM-head units (percent) left to dynamic claims
// by default.  A claimed tail lets faster SMs take over work from slower ones,
// but on the measured workloads the SMs' end times within a phase differ by only
// 1-3 us, and the claims (an L2 round trip each) cost more than they balance
// (Llama-3.2-1B batch 1: 539 us static, 545 with 10-25 % of the LM head claimed,
// 647 with all three phases at 25 %), so the default assignment is static.
constexpr int kDynPercent = 0;

// claim counters of one step: per layer gate/up and each down K slice, then the LM head
MK_HD inline int n_pools(const Dims& D) { return D.L * (1 + D.n_ks) + 1; }
MK_HD inline int pool_gu(const Dims& D, int layer) { return layer * (1 + D.n_ks); }
MK_HD inline int pool_dn(const Dims& D, int layer, int ks) { return layer * (1 + D.n_ks) + 1 + ks; }
MK_HD inline int pool_lm(const Dims& D) { return D.L * (1 + D.n_ks); }

// lanes the kernel is instantiated for: the batch size rounded up to 1, 2, 4 or 8
MK_HD inline int lanes_template(int nb) { return nb <= 1 ? 1 : nb <= 2 ? 2 : nb <= 4 ? 4 : 8; }

MK_HD inline int ctr_layer(int layer, int kind) { return layer * kCountersPerLayer + kind; }
MK_HD inline int ctr_part(const Dims& D, int layer, int b, int g) {
  return D.L * kCountersPerLayer + (layer * kMaxNB + b) * D.Hkv + g;
}
MK_HD inline int ctr_lm(const Dims& D) { return D.L * kCountersPerLayer + D.L * kMaxNB * D.Hkv; }
// steps of the current launch whose greedy ids are written (multi-step launches)
MK_HD inline int ctr_step(const Dims& D) { return ctr_lm(D) + 1; }
MK_HD inline int n_counters(const Dims& D) { return ctr_lm(D) + 2; }

// attention unit i = (lane * Hkv + kv head) * S + slice
MK_HD inline void attn_unit(uint32_t i, int Hkv, int S, int* b, int* g, int* s) {
  *s = (int)(i % (uint32_t)S);
  const uint32_t bg = i / (uint32_t)S;
  *g = (int)(bg % (uint32_t)Hkv);
  *b = (int)(bg / (uint32_t)Hkv);
}

// Shape derivation and tape lowering (mk_sched.cpp).
std::string derive_dims(int n_layers, int hidden, int n_heads, int n_kv_heads, int head_dim,
                        int ffn, int vocab, int tied, float eps, int max_batch, int max_seq,
                        int n_sm, Dims* out);
int attn_slices(const Dims& D, int n_sm, int nb);
// dyn_percent: share of the gate/up, down and LM-head units claimed at run time
// (0: every unit statically assigned)
Tape lower(const Dims& D, int n_sm, int nb, int dyn_percent = kDynPercent, int region = REGION_ALL);

struct SimReport {
  bool deadlock_free = false, coverage_ok = false, targets_ok = false;
  int max_instr_per_sm = 0, n_instr_total = 0;
  int64_t bytes_min = 0, bytes_max = 0;
  std::string error;
};
SimReport simulate(const Dims& D, int n_sm, const Tape& t);

// Dynamic shared memory layout of the kernel.
struct SmemLayout {
  int ring_pages;
  int act_bytes;     // activation / attention scratch region
  int bar_off;       // mbarriers
  int misc_off;      // small reduction scratch
  int total;
};
SmemLayout smem_layout(const Dims& D, int nb_max, int max_dyn_smem, int want_pages);

}  // namespace mk
