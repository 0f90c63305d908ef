// mk_kernel.cuh -- the persistent decode megakernel (sm_100a).
//
// One launch = one decode step of the whole model.  Grid = one CTA per SM
// (cooperative launch, so all CTAs are co-resident), 288 threads:
//   warp 0, lane 0   producer: walks this SM's tape and streams every unit's
//                    weights (or KV pages) into a ring of 16 KiB shared-memory
//                    pages with bulk copies, running ahead of the consumers and
//                    across instruction boundaries -- weights do not depend on
//                    activations, so they are fetched while the consumers are
//                    still waiting on a counter (the "paged shared memory" of
//                    the Hazy megakernel article, section "Megakernel: a
//                    deep-fusion design from scratch");
//   warps 1..8       consumers: for each instruction wait on its counter, stage
//                    the activation vector (with RMSNorm where the op fuses
//                    it), then each warp takes whole pages (units), computes
//                    the bf16 x fp32 matvec on CUDA cores and runs the op's
//                    epilogue, and bumps the op's counter when its pages are
//                    done (the completion counters of the same article).
//
// Publishing activations without a fence.  Inside a step every activation
// element (q, the new K/V row, the attention output, the residual after the O
// projection, the SwiGLU product, each down-projection K slice) is written
// exactly once, into a buffer that holds a sentinel NaN until then.  Readers
// check every element they load and re-read the ones that still hold the
// sentinel, so a value is trusted by what it is, not by the order it became
// visible in: the counters are only hints that tell a waiting SM when to start
// reading (relaxed increments and polls), and no release fence -- which costs
// microseconds per phase under a full HBM stream -- sits on the layer chain.
// Buffers alternate between two sets by decode step; during step t every SM
// refills its share of the other set with the sentinel, after step t - 1 has
// ended everywhere (the step counter below) and before step t + 1 begins.  The
// one acquire/release chain per step is the greedy-id reduction of the LM head
// (acq_rel arrivals, a release of the step counter), which also orders this
// step's KV-cache writes before the next step's bulk copies of them.
//
// Every wait is bounded (globaltimer); on timeout the CTA records an error word,
// raises a global abort flag that every other waiter polls, drains its in-flight
// copies and returns, so a bad tape cannot hang the GPU.
#pragma once

#include <math_constants.h>

#include "mk_device.cuh"
#include "mk_matvec.cuh"
#include "mk_plan.h"
#include "mk_tc.cuh"

namespace mk {

struct LayerW {
  const uint16_t* attn_norm;
  const uint16_t* wq;
  const uint16_t* wk;
  const uint16_t* wv;
  const uint16_t* wo;
  const uint16_t* mlp_norm;
  const uint16_t* w_gate;
  const uint16_t* w_up;
  const uint16_t* w_down;
};

struct ErrWord {
  uint32_t code, sm, instr, info;
  uint32_t abort;
  uint32_t pad[3];
};

enum DevErr : uint32_t {
  E_WAIT_COUNTER = 1,  // a counter did not reach its target in time
  E_WAIT_FULL = 2,     // a ring page did not arrive in time
  E_WAIT_EMPTY = 3,    // a ring page was not released in time
  E_BAD_TOKEN = 4,     // a lane's token was outside [0, vocab) (treated as 0)
  E_DRAIN = 5,         // in-flight copies did not land before exit
  E_WAIT_DATA = 6,     // an activation element was not written in time
};

struct KParams {
  // tape of this step's batch size
  const Instr* instrs;
  const uint32_t* sm_off;
  int S;  // attention slices per (lane, kv head)
  // the embedding table (layer-0 inputs); all other weights are named by the instructions
  const uint16_t* embed;
  // Activations: two sets (by decode-step parity), each L layer blocks of
  // layer_floats floats followed by L accumulators of acc_floats floats.  Inside
  // a block, with MB = max_batch lanes:
  //   off_q   [MB][qdim]      rotated queries
  //   off_kvn [MB][2][kvdim]  this step's K and V rows (fp32, before caching)
  //   off_o   [MB][qdim]      attention output
  //   off_x1  [MB][H]         residual after the O projection
  //   off_a   [MB][F]         silu(gate) * up
  // and the accumulator of layer l, [MB][H] 64-bit counted fixed-point sums
  // (acc_enc), holds the residual after its down projection: x1 plus every K
  // slice's partial, 1 + n_ks terms.  After the accumulators, at claim_off, the
  // claim counters of the step's dynamic tails (uint32, Instr::pool), then at
  // lmkey_off the greedy keys of the step (uint64 per lane, lm_key).  Float
  // blocks refill with the sentinel, the rest with zero.
  float* acts;
  long long set_floats, layer_floats, acc_base, acc_floats, claim_off, lmkey_off;
  int off_q, off_kvn, off_o, off_x1, off_a;
  int parity0;  // set of this launch's step 0
  int hints;    // bit op set: instructions of that op wait on their hint counter before
                // reading their inputs; clear: they read and validate the inputs at once
                // (the inputs carry their own readiness)
  float* part;  // attention partials [8][Hkv][S][rep][d + 2]
  // KV cache [layer][physical page][kv head][K, V][PL][d]: a page's K and V are
  // one contiguous 16 KiB block
  uint16_t* kv;
  const int* page_table;  // [max_batch][pages_per_seq]
  uint32_t* ctr;          // counters of this step
  uint32_t* ctr_next;     // counters of the next step (zeroed here)
  int n_counters;
  ErrWord* err;
  const float2* rope;  // [max_seq][d/2] (cos, sin)
  // steps: n_steps decode steps run in this launch, lane b of step t at position
  // pos[b] + t.  Step t's input tokens: tokens + t * nb when tokens are given
  // for every step (chain == 0), else step 0 reads tokens and step t > 0 reads the
  // ids step t - 1 wrote.  Step t writes its ids to ids + t * ids_stride and, when
  // logits is set, its logits to logits + t * nb * V (logits_last: only the last
  // step, at logits).
  int nb;
  int n_steps;
  int chain;
  int ids_stride;
  int logits_last;
  const int* tokens;
  int pos[kMaxNB];
  int slot[kMaxNB];
  float* logits;
  int* ids;
  unsigned long long wait_limit_ns;
  long long* prof;   // profile records [n_sm][prof_stride][kProfSlots] or null
  int prof_stride;
  // shared memory layout
  int ring_pages, act_off, bar_off, misc_off;
  Dims D;
};

struct Misc {
  // a copy of the launch parameters: producer and consumers read them through a
  // reference, and a generic load of the parameter space is a global-memory load
  KParams kp;
  float red[kConsumerWarps][kMaxNB];
  float lmv[kConsumerWarps][kMaxNB];
  int lmi[kConsumerWarps][kMaxNB];
  int tok[kMaxNB];
  long long warp_done[kConsumerWarps];  // profile mode: when each warp finished its units
  long long warp_entry[kConsumerWarps];  // profile mode: when each warp entered its matvec
  long long warp_first[kConsumerWarps];  // profile mode: when each warp had its first page
  int pos[kMaxNB];       // each lane's position in the current step
  int step;              // the current step of this launch
  int cur_phys[kMaxNB];  // physical KV page holding each lane's position this step
  float2 rope_cs[kMaxNB][64];  // (cos, sin) of each lane's position, per frequency
  float* actset;         // the activation set of the current step
  uint32_t i0;           // this SM's first tape index (profile records)
  uint32_t n_instr;      // this SM's tape length
  uint32_t attn_extra;   // attention signals beyond one per (lane, kv head), summed over this launch's steps
  unsigned int slow_n;   // profile mode: group re-reads of unwritten activations
  unsigned long long slow_ns;  // and the time they took (summed over threads)
  long long t_stage_in, t_stage_loaded;  // profile mode: stage entry, thread 0's loads back
  long long t_sum_x1, t_sum_p;           // profile mode: residual sum, x1 back, partials back
  volatile int stop;
  volatile int last;
  uint32_t issued;  // pages the ring producer issued
  // Dynamic tails.  unit[slot]: the unit whose weights the page in that ring slot
  // holds (written by the producer before the page's full-barrier arrival).
  // dyn_end[s & 15]: for the s-th instruction of this launch (s = step * tape
  // length + index), (s << 32) | the stream position where its pages end, written
  // by the producer once its claims are exhausted.  cons_seq: the instruction the
  // consumers are in (the producer reuses an entry only after they left it).
  uint32_t unit[64];
  volatile unsigned long long dyn_end[16];
  volatile uint32_t cons_seq;
  volatile uint32_t last_claim;
  int entry_abort;
  // Tensor-core units (8-lane kernel of the Llama-3.2-1B shape family): the two
  // accumulators in tensor memory (written: tc_accf, read back: tc_acce) and the
  // tensor-memory base address.
  uint64_t tc_accf[2], tc_acce[2];
  uint32_t tmem_base;
};
// the misc region is what smem_layout leaves after the barriers: 8192 - 8 * (128 + 64)
static_assert(sizeof(Misc) <= 8192 - 8 * (128 + 64), "Misc does not fit its shared-memory region");

// ---------------------------------------------------------------- errors & waits

__device__ __forceinline__ bool aborted(const KParams& p) { return ld_relaxed_u32(&p.err->abort) != 0; }

static __device__ __noinline__ void raise_error(const KParams& p, uint32_t code, uint32_t instr, uint32_t info,
                                         bool abort) {
  if (atomicCAS(&p.err->code, 0u, code) == 0u) {
    p.err->sm = blockIdx.x;
    p.err->instr = instr;
    p.err->info = info;
  }
  __threadfence();
  if (abort) atomicExch(&p.err->abort, 1u);
}

// Spin until *c >= target (acquire), the abort flag rises, or the time limit passes.
static __device__ __noinline__ bool wait_counter(const KParams& p, const uint32_t* c, uint32_t target,
                                          uint32_t instr) {
  if (ld_acquire_u32(c) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_u32(c) >= target) return true;
    if ((it & 63) == 0) {
      if (aborted(p)) return false;
      if (globaltimer_ns() - t0 > p.wait_limit_ns) {
        raise_error(p, E_WAIT_COUNTER, instr, target, true);
        return false;
      }
    }
    if (it > 512) __nanosleep(32);
  }
}

// Spin until the hint counter *c reaches target (relaxed: the data it announces
// is validated element by element), the abort flag rises, or the time passes.
static __device__ __noinline__ bool wait_hint(const KParams& p, const uint32_t* c, uint32_t target, uint32_t instr) {
  if (ld_relaxed_u32(c) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ld_relaxed_u32(c) >= target) return true;
    if ((it & 63) == 0) {
      if (aborted(p)) return false;
      if (globaltimer_ns() - t0 > p.wait_limit_ns) {
        raise_error(p, E_WAIT_COUNTER, instr, target, true);
        return false;
      }
    }
    if (it > 512) __nanosleep(32);
  }
}

// Re-read an activation element group until no element holds the sentinel
// (bounded; on timeout or abort the CTA stops and zeros are returned).
static __device__ __noinline__ float4 poll4_slow(const KParams& p, const float* src, uint32_t instr, Misc* misc) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    const float4 v = ld_relaxed_f4(src);
    if (!any_sent(v)) return v;
    if ((it & 63) == 0) {
      if (aborted(p)) break;
      if (globaltimer_ns() - t0 > p.wait_limit_ns) {
        raise_error(p, E_WAIT_DATA, instr, 4, true);
        break;
      }
    }
  }
  misc->stop = 1;
  return make_float4(0.f, 0.f, 0.f, 0.f);
}
static __device__ __noinline__ float2 poll2_slow(const KParams& p, const float* src, uint32_t instr, Misc* misc) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    const float2 v = ld_relaxed_f2(src);
    if (!any_sent(v)) return v;
    if ((it & 63) == 0) {
      if (aborted(p)) break;
      if (globaltimer_ns() - t0 > p.wait_limit_ns) {
        raise_error(p, E_WAIT_DATA, instr, 2, true);
        break;
      }
    }
  }
  misc->stop = 1;
  return make_float2(0.f, 0.f);
}
static __device__ __noinline__ float poll1_slow(const KParams& p, const float* src, uint32_t instr, Misc* misc) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    const float v = ld_relaxed_f1(src);
    if (!is_sent(v)) return v;
    if ((it & 63) == 0) {
      if (aborted(p)) break;
      if (globaltimer_ns() - t0 > p.wait_limit_ns) {
        raise_error(p, E_WAIT_DATA, instr, 1, true);
        break;
      }
    }
  }
  misc->stop = 1;
  return 0.f;
}
// Bookkeeping of a group re-read: true while the group may be read again;
// false (CTA stopped, error raised on timeout) once it may not.
struct Spin {
  uint64_t t0 = 0, tp = 0;
  uint32_t it = 0;
  const KParams* pp;
  Misc* m;
  // profile mode: lane 0 of each warp counts its re-read groups and their time
  // (one shared-memory atomic per warp, so that profiling barely slows the wait)
  __device__ __forceinline__ Spin(const KParams& p, Misc* misc) : pp(&p), m(misc) {
    if (p.prof && (threadIdx.x & 31) == 0) {
      tp = globaltimer_ns();
      atomicAdd(&misc->slow_n, 1u);
    }
  }
  __device__ __forceinline__ ~Spin() {
    if (pp->prof && (threadIdx.x & 31) == 0) atomicAdd(&m->slow_ns, (unsigned long long)(globaltimer_ns() - tp));
  }
  __device__ __forceinline__ bool again(const KParams& p, uint32_t instr, uint32_t info, Misc* misc) {
    ++it;
    if ((it & 15) == 0) {
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      if (aborted(p)) { misc->stop = 1; return false; }
      if (now - t0 > p.wait_limit_ns) {
        raise_error(p, E_WAIT_DATA, instr, info, true);
        misc->stop = 1;
        return false;
      }
    }
    if (it > 64) __nanosleep(32);
    return true;
  }
};

// fast path: the caller issues its loads first, then validates each
__device__ __forceinline__ void ready(float4& v, const KParams& p, const float* src, uint32_t instr, Misc* misc) {
  if (any_sent(v)) v = poll4_slow(p, src, instr, misc);
}
__device__ __forceinline__ void ready(float2& v, const KParams& p, const float* src, uint32_t instr, Misc* misc) {
  if (any_sent(v)) v = poll2_slow(p, src, instr, misc);
}
__device__ __forceinline__ void ready(float& v, const KParams& p, const float* src, uint32_t instr, Misc* misc) {
  if (is_sent(v)) v = poll1_slow(p, src, instr, misc);
}

// Wait for an mbarrier phase.  The abort flag (an L2 load) and the clock are
// only consulted once a wait has lasted a while, so a page that lands during a
// short wait is seen at once.  honor_abort = false is used by the exit drain,
// which must wait for copies in flight even after an abort.
__device__ __forceinline__ bool wait_mbar(const KParams& p, uint64_t* bar, uint32_t parity,
                                          uint32_t code, uint32_t instr, bool honor_abort) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255) == 0) {
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      if (honor_abort && aborted(p)) return false;
      if (now - t0 > p.wait_limit_ns) {
        raise_error(p, code, instr, parity, true);
        return false;
      }
    }
  }
}

// Slices actually used for a (lane, kv head) with npg KV pages: about one per
// two pages, at most the tape's S.  A short context is then one slice, which
// writes its output directly instead of through partials and a merge.
__device__ __forceinline__ int attn_slices_used(int S, int npg) { return max(1, min(S, npg / 2)); }

// What attention unit (lane, kv head, slice s) does at a context of npg pages.
// Short contexts (at most kHeadSplitPages pages) with S >= rep split the group
// by query head instead: slice s < rep takes query head s of the group over all
// pages and writes it directly, so rep SMs share the group's latency and no
// merge is needed (the pages are read rep times, from L2 after the first).
// Longer contexts split the pages into se slices of all rep heads.
constexpr int kHeadSplitPages = 4;
struct AttnPlan {
  bool active, single;  // single: one query head (head split)
  int head, pb, pe, se;  // head: first query head within the group; pages [pb, pe)
};
__device__ __forceinline__ AttnPlan attn_plan(int S, int rep, int npg, int s) {
  AttnPlan a;
  if (rep > 1 && S >= rep && npg <= kHeadSplitPages) {
    a.single = true;
    a.active = s < rep;
    a.head = s;
    a.pb = 0;
    a.pe = npg;
    a.se = 1;
  } else {
    a.single = false;
    a.se = attn_slices_used(S, npg);
    a.active = s < a.se;
    a.head = 0;
    a.pb = (int)((long long)s * npg / a.se);
    a.pe = (int)((long long)(s + 1) * npg / a.se);
  }
  return a;
}

// ---------------------------------------------------------------- dynamic tails

// Producer: wait until the consumers have entered instruction seq - 15, so the
// dyn_end entry of seq - 16 is no longer read.
static __device__ __noinline__ bool wait_consumers(const KParams& p, Misc* misc, uint32_t seq, uint32_t instr) {
  if (misc->cons_seq + 16u > seq) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (misc->cons_seq + 16u > seq) return true;
    if ((it & 63) == 0) {
      if (aborted(p)) return false;
      if (globaltimer_ns() - t0 > p.wait_limit_ns) {
        raise_error(p, E_WAIT_EMPTY, instr, seq, true);
        return false;
      }
    }
    __nanosleep(64);
  }
}

// Consumer: wait for the page at stream position q of a dynamic instruction
// (launch-wide index seq).  1: the page is there and belongs to the instruction;
// 0: the instruction's pages ended before q (the page at q, if any, is the next
// instruction's and stays untouched); -1: aborted or timed out.  The end is read
// again after the barrier completes: the producer publishes it before issuing
// any later instruction's page, so a completed foreign page implies a visible end.
__device__ __forceinline__ int wait_dyn(const KParams& p, uint64_t* bar, uint32_t parity, Misc* misc,
                                        uint32_t seq, uint32_t q, uint32_t instr) {
  const volatile unsigned long long* de = &misc->dyn_end[seq & 15];
  auto ended = [&]() {
    const unsigned long long e = *de;
    return (uint32_t)(e >> 32) == seq && (int32_t)(q - (uint32_t)e) >= 0;
  };
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (ended()) return 0;
    if (mbar_try_wait_hint(bar, parity, 256u)) return ended() ? 0 : 1;
    if ((it & 63) == 63) {
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      if (aborted(p)) return -1;
      if (now - t0 > p.wait_limit_ns) {
        raise_error(p, E_WAIT_FULL, instr, q, true);
        return -1;
      }
    }
  }
}

// ---------------------------------------------------------------- producer

__device__ __forceinline__ void issue_matvec_page(const KParams& p, const Instr& I, uint32_t u,
                                                  uint8_t* dst, uint64_t* bar, uint64_t pol) {
  const Dims& D = p.D;
  switch (I.op) {
    case OP_QKV: {  // packed: the unit's RP first-half rows, then its RP second-half rows
      const uint32_t bytes = (uint32_t)(2 * D.RP) * D.H * 2;
      mbar_arrive_expect_tx(bar, bytes);
      bulk_g2s(dst, static_cast<const uint16_t*>(I.ptr[0]) + (size_t)u * (2 * D.RP) * D.H, bytes, bar, pol);
      break;
    }
    case OP_O: {
      const int r0 = (int)u * D.Ro, nr = min(D.Ro, D.H - r0);
      const uint32_t bytes = (uint32_t)nr * D.qdim * 2;
      mbar_arrive_expect_tx(bar, bytes);
      bulk_g2s(dst, static_cast<const uint16_t*>(I.ptr[0]) + (size_t)r0 * D.qdim, bytes, bar, pol);
      break;
    }
    case OP_GU: {  // packed: Rgu gate rows, then the same Rgu up rows (zero past ffn)
      const uint32_t bytes = (uint32_t)(2 * D.Rgu) * D.H * 2;
      mbar_arrive_expect_tx(bar, bytes);
      bulk_g2s(dst, static_cast<const uint16_t*>(I.ptr[0]) + (size_t)u * (2 * D.Rgu) * D.H, bytes, bar, pol);
      break;
    }
    case OP_DOWN: {  // packed K-slice major: the unit's rows of slice I.arg are adjacent
      const int r0 = (int)u * D.Rdn, nr = min(D.Rdn, D.H - r0);
      const uint32_t bytes = (uint32_t)nr * D.KS * 2;
      const uint16_t* w = static_cast<const uint16_t*>(I.ptr[0]) + ((size_t)I.arg * D.H + r0) * D.KS;
      mbar_arrive_expect_tx(bar, bytes);
      bulk_g2s(dst, w, bytes, bar, pol);
      break;
    }
    case OP_LM: {
      const int r0 = (int)u * D.Rlm, nr = min(D.Rlm, D.V - r0);
      const uint32_t bytes = (uint32_t)nr * D.H * 2;
      mbar_arrive_expect_tx(bar, bytes);
      bulk_g2s(dst, static_cast<const uint16_t*>(I.ptr[0]) + (size_t)r0 * D.H, bytes, bar, pol);
      break;
    }
  }
}

// The producer walks this SM's tape and issues every unit's page in order.  It
// touches global memory only for the tape (the next instruction is loaded while
// the current one is issued) and the page table; every other address comes from
// the instruction, so the issue loop never stalls on a dependent load.
static __device__ __noinline__ void producer(const KParams& p, uint8_t* ring, uint64_t* full, uint64_t* empty,
                                      Misc* misc) {
  const Dims& D = p.D;
  const uint32_t NP = (uint32_t)p.ring_pages;
  const uint64_t pol = l2_evict_first_policy();
  const uint32_t i0 = p.sm_off[blockIdx.x], i1 = p.sm_off[blockIdx.x + 1];
  uint32_t pidx = 0;
  RingPos rp;
  rp.init(0, NP);
  bool ok = true;
  for (int t = 0; t < p.n_steps && ok; ++t) {
  Instr I;
  if (i0 < i1) I = p.instrs[i0];
  bool synced = false;  // this step's claim counters are ready (step t - 1 ended)
  for (uint32_t ii = i0; ii < i1 && ok; ++ii) {
    const Instr In = ii + 1 < i1 ? p.instrs[ii + 1] : I;
    long long* rec = p.prof ? p.prof + ((size_t)blockIdx.x * p.prof_stride + (ii - i0)) * kProfSlots : nullptr;
    long long acc_wait = 0, acc_pages = 0;
    if (rec) rec[5] = (long long)globaltimer_ns();
    if (I.op == OP_ATTN) {
      // KV pages of step t hold the positions earlier steps of this launch wrote:
      // copy them only once step t - 1 has ended (its greedy ids are out, which
      // every SM's KV writes of that step precede).  By then this producer has
      // issued every page of the earlier steps, so the wait cannot hold up the
      // consumers it depends on.
      if (t > 0) {
        if (!(ok = wait_counter(p, p.ctr + ctr_step(D), (uint32_t)t, ii))) break;
        fence_proxy_async_global();  // the bulk copies below read what the acquire made visible
      }
      for (uint32_t k = 0; k < I.n_units && ok; ++k) {
        int b, g, s;
        attn_unit(I.u0 + k, D.Hkv, p.S, &b, &g, &s);
        const int pos = p.pos[b] + t, npg = pos / D.PL + 1;
        const AttnPlan ap = attn_plan(p.S, D.rep, npg, s);
        if (!ap.active) continue;
        const int pb = ap.pb, pe = ap.pe;
        const int* pt = p.page_table + p.slot[b] * D.pages_per_seq;
        int phys_next = pb < pe ? pt[pb] : 0;
        for (int j = pb; j < pe; ++j) {
          const int phys = phys_next;
          if (j + 1 < pe) phys_next = pt[j + 1];  // in flight while this page is issued
          if (!(ok = wait_mbar(p, &empty[rp.slot], rp.sphase ^ 1u, E_WAIT_EMPTY, ii, true))) break;
          // only positions written by earlier steps; the current one is patched in by the consumer
          const int n_old = min(D.PL, pos - j * D.PL);
          uint64_t* fb = &full[rp.fidx];
          if (n_old > 0) {
            const size_t kvp = (size_t)D.PL * D.d;  // elements of one page's K (or V)
            const uint16_t* src = p.kv + (((size_t)I.layer * D.n_phys_pages + phys) * D.Hkv + g) * 2 * kvp;
            uint8_t* dst = ring + (size_t)rp.slot * kPageBytes;
            if (n_old == D.PL) {  // a full page: K and V in one copy
              mbar_arrive_expect_tx(fb, (uint32_t)(4 * kvp));
              bulk_g2s(dst, src, (uint32_t)(4 * kvp), fb, pol);
            } else {  // the written positions of K, then of V
              const uint32_t bytes = (uint32_t)n_old * D.d * 2;
              mbar_arrive_expect_tx(fb, 2 * bytes);
              bulk_g2s(dst, src, bytes, fb, pol);
              bulk_g2s(dst + 2 * kvp, src + kvp, bytes, fb, pol);
            }
          } else {
            mbar_arrive(fb);
          }
          ++pidx;
          rp.advance(1, NP);
        }
      }
    } else if (I.op == OP_GU_TC || I.op == OP_LM_TC) {
      // a unit is a 128-row block: its nkt K tiles, each one contiguous 16 KiB tile
      const uint16_t* base = static_cast<const uint16_t*>(I.ptr[0]);
      for (uint32_t k = 0; k < I.n_units && ok; ++k)
        for (int kt = 0; kt < D.nkt && ok; ++kt) {
          if (!(ok = wait_mbar(p, &empty[rp.slot], rp.sphase ^ 1u, E_WAIT_EMPTY, ii, true))) break;
          mbar_arrive_expect_tx(&full[rp.fidx], (uint32_t)kPageBytes);
          bulk_g2s(ring + (size_t)rp.slot * kPageBytes,
                   base + ((size_t)(I.u0 + k) * D.nkt + kt) * (kPageBytes / 2), (uint32_t)kPageBytes,
                   &full[rp.fidx], pol);
          ++pidx;
          rp.advance(1, NP);
        }
    } else {
      // The static units, then (dynamic tail) the chunks this SM claims from the
      // phase's pool.  Three claims are in flight at a time (the first one issued
      // under the last static pages), so a claim's round trip stays hidden behind
      // the stream.  Claims are used in the order issued, so their values grow and
      // the first one past the pool ends the instruction.
      uint32_t* claim = nullptr;
      uint32_t chunk = 0, pn = 0, va = 0, vb = 0, vc = 0;
      if (I.pool) {
        // the counters live in this step's activation set, which SMs zeroed
        // during step t - 1: wait until every SM is past that step
        if (t > 0 && !synced) {
          if (!(ok = wait_counter(p, p.ctr + ctr_step(D), (uint32_t)t, ii))) break;
          synced = true;
        }
        claim = reinterpret_cast<uint32_t*>(p.acts + (size_t)((p.parity0 + t) & 1) * p.set_floats + p.claim_off) +
                ((I.pool & 0xFFFFFFu) - 1u);
        chunk = I.pool >> 24;
        pn = I.pool_u1 - I.pool_u0;
      }
      auto page = [&](uint32_t u) {
        const long long tw = rec ? (long long)globaltimer_ns() : 0;
        if (!(ok = wait_mbar(p, &empty[rp.slot], rp.sphase ^ 1u, E_WAIT_EMPTY, ii, true))) return;
        if (rec) { acc_wait += (long long)globaltimer_ns() - tw; acc_pages += 1; }
        misc->unit[rp.slot] = u;  // published to the consumer by the full barrier's arrival
        issue_matvec_page(p, I, u, ring + (size_t)rp.slot * kPageBytes, &full[rp.fidx], pol);
        ++pidx;
        rp.advance(1, NP);
      };
      const uint32_t k_claim = I.n_units > 4u ? I.n_units - 4u : 0u;
      for (uint32_t k = 0; k < I.n_units && ok; ++k) {
        if (claim && k == k_claim) va = atomicAdd(claim, chunk);
        page(I.u0 + k);
      }
      if (I.pool && ok) {
        if (I.n_units == 0) va = atomicAdd(claim, chunk);
        vb = atomicAdd(claim, chunk);
        vc = atomicAdd(claim, chunk);
        auto take = [&](uint32_t& v) {  // stream claim v's chunk, then claim again into v
          if (v >= pn) return false;
          const uint32_t ve = min(v + chunk, pn);
          for (uint32_t x = v; x < ve && ok; ++x) page(I.pool_u0 + x);
          v = atomicAdd(claim, chunk);
          return ok;
        };
        while (take(va) && take(vb) && take(vc)) {
        }
        misc->last_claim = va + vb + vc;  // every claim has landed before the step can end
        // publish where this instruction's pages end; its entry's previous user
        // (instruction seq - 16) must be behind the consumers
        const uint32_t seq = (uint32_t)t * (i1 - i0) + (ii - i0);
        if (ok) ok = wait_consumers(p, misc, seq, ii);
        if (ok) misc->dyn_end[seq & 15] = ((unsigned long long)seq << 32) | pidx;
      }
    }
    if (rec) { rec[6] = (long long)globaltimer_ns(); rec[9] += acc_wait; rec[10] += acc_pages; }
    I = In;
  }
  }
  misc->issued = pidx;
  // every copy issued must land before the CTA exits (also after an abort)
  const uint32_t first = pidx > NP ? pidx - NP : 0;
  for (uint32_t q = first; q < pidx; ++q)
    if (!wait_mbar(p, &full[q % (2 * NP)], (q / (2 * NP)) & 1, E_DRAIN, q, false)) break;
}

// ---------------------------------------------------------------- consumers: staging

// Slow paths of the staging: some element of the chunk still held the
// sentinel, so the whole group of loads is issued again (in parallel) until
// every element is written.  Results come back by value: a fast-path variable
// whose address escaped would live in local memory and serialise its loads.
template <int NBT>
struct Chunk8 {
  float4 l[NBT], h[NBT];
};
template <int NBT>
static __device__ __noinline__ Chunk8<NBT> stage_one_slow(const KParams& p, const float* src, int ld, uint32_t ii,
                                                   Misc* misc) {
  Chunk8<NBT> r;
  Spin sp(p, misc);
  do {
    bool bad = false;
#pragma unroll
    for (int b = 0; b < NBT; ++b) {
      r.l[b] = r.h[b] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (b < p.nb) {
        r.l[b] = ld_relaxed_f4(src + (size_t)b * ld);
        r.h[b] = ld_relaxed_f4(src + (size_t)b * ld + 4);
      }
    }
#pragma unroll
    for (int b = 0; b < NBT; ++b) bad |= any_sent(r.l[b]) | any_sent(r.h[b]);
    if (!bad) return r;
  } while (sp.again(p, ii, 8, misc));
#pragma unroll
  for (int b = 0; b < NBT; ++b) r.l[b] = r.h[b] = make_float4(0.f, 0.f, 0.f, 0.f);
  return r;
}
// one 8-element chunk of each lane's residual accumulator, until all 1 + n_ks terms are in
template <int NBT>
static __device__ __noinline__ Chunk8<NBT> acc_chunk_slow(const KParams& p, const unsigned long long* src, int ld,
                                                   uint32_t ii, Misc* misc) {
  Chunk8<NBT> r;
  const uint32_t want = 1u + (uint32_t)p.D.n_ks;
  Spin sp(p, misc);
  do {
    bool bad = false;
#pragma unroll
    for (int b = 0; b < NBT; ++b) {
      r.l[b] = r.h[b] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (b >= p.nb) continue;
      const ulonglong2 e0 = ld_relaxed_u64x2(src + (size_t)b * ld), e1 = ld_relaxed_u64x2(src + (size_t)b * ld + 2);
      const ulonglong2 e2 = ld_relaxed_u64x2(src + (size_t)b * ld + 4), e3 = ld_relaxed_u64x2(src + (size_t)b * ld + 6);
      bad |= (acc_count(e0.x) != want) | (acc_count(e0.y) != want) | (acc_count(e1.x) != want) |
             (acc_count(e1.y) != want) | (acc_count(e2.x) != want) | (acc_count(e2.y) != want) |
             (acc_count(e3.x) != want) | (acc_count(e3.y) != want);
      r.l[b] = make_float4(acc_value(e0.x), acc_value(e0.y), acc_value(e1.x), acc_value(e1.y));
      r.h[b] = make_float4(acc_value(e2.x), acc_value(e2.y), acc_value(e3.x), acc_value(e3.y));
    }
    if (!bad) return r;
  } while (sp.again(p, ii, 9, misc));
#pragma unroll
  for (int b = 0; b < NBT; ++b) r.l[b] = r.h[b] = make_float4(0.f, 0.f, 0.f, 0.f);
  return r;
}

// Stage NBT activation rows of length K into shared memory in the split layout
// used by the matvec (chunk c of lane b: elements 8c..8c+3 at lo[b*nch + c],
// 8c+4..8c+7 at hi[b*nch + c]).  Sources (MODE):
//   ST_EMB  the bf16 embedding rows of the lanes' tokens (layer 0);
//   ST_ONE  one fp32 vector per lane at src + b * ld;
//   ST_ACC  the residual after a down projection: the layer's accumulator at
//           src (64-bit elements, lane stride ld).
// The other sources are this step's activations: every element is validated
// (sentinel, or the accumulator's term count) and re-read until written.  NORM
// applies RMSNorm with the bf16 gain.  Lanes >= nb are zero.
enum { ST_EMB = 0, ST_ONE = 1, ST_ACC = 2 };

// BOP: write the staged values instead as the tensor cores' B operand (8 lanes,
// K-major, 128-byte swizzle): row b the bf16 high part of lane b, row 8 + b the low
// part, one 2 KiB tile per 64 K (16 rows x 128 bytes, 8-row groups 1 KiB apart).
template <int NBT, int MODE, bool NORM, bool BOP = false>
__device__ __forceinline__ void stage(const KParams& p, float* act, Misc* misc, const float* src, int ld,
                                      int K, const uint16_t* gain, uint32_t ii) {
  static_assert(!BOP || NBT == 8, "the B operand holds 8 lanes");
  const int ct = threadIdx.x - 32, cw = ct >> 5, lane = ct & 31;
  const int nch = K >> 3;
  float4* lo = reinterpret_cast<float4*>(act);
  float4* hi = lo + NBT * nch;
  if (p.prof && ct == 0) misc->t_stage_in = (long long)globaltimer_ns();
  float ss[NBT];
#pragma unroll
  for (int b = 0; b < NBT; ++b) ss[b] = 0.f;
  for (int c = ct; c < nch; c += 256) {
    float g[8];
    if (NORM) {  // the gain is applied here; the 1/rms scale after the reduction
      const uint4 gw = ldnc16(gain + c * 8);
      g[0] = bf_lo(gw.x); g[1] = bf_hi(gw.x); g[2] = bf_lo(gw.y); g[3] = bf_hi(gw.y);
      g[4] = bf_lo(gw.z); g[5] = bf_hi(gw.z); g[6] = bf_lo(gw.w); g[7] = bf_hi(gw.w);
    }
    float4 vl[NBT], vh[NBT];
    if constexpr (MODE == ST_EMB) {
#pragma unroll
      for (int b = 0; b < NBT; ++b) {
        if (b < p.nb) {
          const uint4 w = ldnc16(p.embed + (size_t)misc->tok[b] * p.D.H + c * 8);
          vl[b] = make_float4(bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
          vh[b] = make_float4(bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w));
        } else {
          vl[b] = vh[b] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    } else if constexpr (MODE == ST_ONE) {
#pragma unroll
      for (int b = 0; b < NBT; ++b) {  // issue every load, then validate
        if (b < p.nb) {
          vl[b] = ld_relaxed_f4(src + (size_t)b * ld + c * 8);
          vh[b] = ld_relaxed_f4(src + (size_t)b * ld + c * 8 + 4);
        } else {
          vl[b] = vh[b] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      bool bad = false;
#pragma unroll
      for (int b = 0; b < NBT; ++b) bad |= any_sent(vl[b]) | any_sent(vh[b]);
      if (bad) {
        const Chunk8<NBT> r = stage_one_slow<NBT>(p, src + c * 8, ld, ii, misc);
#pragma unroll
        for (int b = 0; b < NBT; ++b) { vl[b] = r.l[b]; vh[b] = r.h[b]; }
      }
    } else {  // ST_ACC: src is the accumulator array
      const unsigned long long* A = reinterpret_cast<const unsigned long long*>(src) + c * 8;
      const uint32_t want = 1u + (uint32_t)p.D.n_ks;
      bool bad = false;
#pragma unroll
      for (int b = 0; b < NBT; ++b) {
        vl[b] = vh[b] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (b >= p.nb) continue;
        const ulonglong2 e0 = ld_relaxed_u64x2(A + (size_t)b * ld), e1 = ld_relaxed_u64x2(A + (size_t)b * ld + 2);
        const ulonglong2 e2 = ld_relaxed_u64x2(A + (size_t)b * ld + 4), e3 = ld_relaxed_u64x2(A + (size_t)b * ld + 6);
        bad |= (acc_count(e0.x) != want) | (acc_count(e0.y) != want) | (acc_count(e1.x) != want) |
               (acc_count(e1.y) != want) | (acc_count(e2.x) != want) | (acc_count(e2.y) != want) |
               (acc_count(e3.x) != want) | (acc_count(e3.y) != want);
        vl[b] = make_float4(acc_value(e0.x), acc_value(e0.y), acc_value(e1.x), acc_value(e1.y));
        vh[b] = make_float4(acc_value(e2.x), acc_value(e2.y), acc_value(e3.x), acc_value(e3.y));
      }
      if (p.prof && ct == 0) {  // when the accumulator came back (profile only)
        misc->t_sum_x1 = (long long)globaltimer_ns() + (bad ? 1 : 0);
        misc->t_sum_p = misc->t_sum_x1;
      }
      if (bad) {
        const Chunk8<NBT> r = acc_chunk_slow<NBT>(p, A, ld, ii, misc);
#pragma unroll
        for (int b = 0; b < NBT; ++b) { vl[b] = r.l[b]; vh[b] = r.h[b]; }
      }
    }
    if (p.prof && ct == 0 && c == 0) {  // the branch waits for the loaded value, then the clock is read
      if (__float_as_uint(vl[0].x) == 0x7FC00001u) misc->slow_n += 0u;
      misc->t_stage_loaded = (long long)globaltimer_ns();
    }
#pragma unroll
    for (int b = 0; b < NBT; ++b) {
      float v[8] = {vl[b].x, vl[b].y, vl[b].z, vl[b].w, vh[b].x, vh[b].y, vh[b].z, vh[b].w};
      if (NORM) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ss[b] = fmaf(v[e], v[e], ss[b]);
          v[e] *= g[e];
        }
      }
      if constexpr (BOP) {
        uint16_t h8[8], l8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) split_bf16(v[e], h8[e], l8[e]);
        uint8_t* tile = reinterpret_cast<uint8_t*>(act) + (size_t)(c >> 3) * 2048;
        const int cs = ((c & 7) ^ (b & 7)) << 4;
        *reinterpret_cast<uint4*>(tile + (b & 7) * 128 + cs) = *reinterpret_cast<const uint4*>(h8);
        *reinterpret_cast<uint4*>(tile + 1024 + (b & 7) * 128 + cs) = *reinterpret_cast<const uint4*>(l8);
      } else {
        lo[b * nch + c] = make_float4(v[0], v[1], v[2], v[3]);
        hi[b * nch + c] = make_float4(v[4], v[5], v[6], v[7]);
      }
    }
  }
  if constexpr (BOP) fence_proxy_async_smem();  // the tensor cores read the operand through the async proxy
  if (NORM) {
#pragma unroll
    for (int b = 0; b < NBT; ++b) {
      float t = ss[b];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
      if (lane == 0) misc->red[cw][b] = t;
    }
    // the 1/rms scale is applied to the matvec outputs (norm_scales), which is
    // the same linear map and saves a pass over the staged vector
  }
  cbar();
}

// ---------------------------------------------------------------- consumers: matvec

// The residual entering layer `layer` at (lane b, row): the embedding for
// layer 0, else the previous layer's accumulator.  The load is issued here;
// resid_finish validates it (all 1 + n_ks terms in) once the value is needed.
struct ResidIn {
  unsigned long long acc;
  const unsigned long long* src;  // null: layer 0, the value is in emb
  float emb;
};
__device__ __forceinline__ const unsigned long long* acc_of(const KParams& p, const Misc* misc, int layer) {
  return reinterpret_cast<const unsigned long long*>(misc->actset + p.acc_base + (size_t)layer * p.acc_floats);
}
__device__ __forceinline__ void resid_issue(const KParams& p, const Misc* misc, int layer, int b, int row,
                                            ResidIn& r) {
  if (layer == 0) {
    r.src = nullptr;
    r.emb = __uint_as_float((uint32_t)p.embed[(size_t)misc->tok[b] * p.D.H + row] << 16);
    return;
  }
  r.src = acc_of(p, misc, layer - 1) + (size_t)b * p.D.H + row;
  r.acc = ld_relaxed_u64(r.src);
}
static __device__ __noinline__ unsigned long long resid_slow(const KParams& p, Misc* misc, const unsigned long long* src,
                                                      uint32_t ii) {
  const uint32_t want = 1u + (uint32_t)p.D.n_ks;
  Spin sp(p, misc);
  do {
    const unsigned long long a = ld_relaxed_u64(src);
    if (acc_count(a) == want) return a;
  } while (sp.again(p, ii, 10, misc));
  return 0ull;
}
__device__ __forceinline__ float resid_finish(const KParams& p, Misc* misc, ResidIn& r, uint32_t ii) {
  if (!r.src) return r.emb;
  if (acc_count(r.acc) != 1u + (uint32_t)p.D.n_ks) r.acc = resid_slow(p, misc, r.src, ii);
  return acc_value(r.acc);
}

__device__ __forceinline__ bool lm_better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// (value, row) as one 64-bit key whose unsigned order is lm_better's order, so an
// atomic maximum over the keys picks the greedy token: the value's bits made
// monotone (negative floats reversed, +0 and -0 equal), then the row reversed so
// the lower row wins a tie.  NaN maps to 0 and never wins, as in lm_better; key 0
// (nothing seen) decodes to row 0x7FFFFFFF.
__device__ __forceinline__ unsigned long long lm_key(float v, int i) {
  if (v != v) return 0ull;
  const uint32_t u = __float_as_uint(v == 0.0f ? 0.0f : v);
  const uint32_t hi = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)hi << 32) | (uint32_t)(0x7FFFFFFF - i);
}
__device__ __forceinline__ int lm_key_row(unsigned long long k) { return 0x7FFFFFFF - (int)(uint32_t)k; }

// 1 / rms of each lane's staged vector (RMSNorm), from the per-warp sums of
// squares the stage left in misc->red.
template <int NBT>
__device__ __forceinline__ void norm_scales(const KParams& p, const Misc* misc, int K, float (&rinv)[NBT]) {
#pragma unroll
  for (int b = 0; b < NBT; ++b) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) t += misc->red[w][b];
    rinv[b] = 1.0f / sqrtf(t / (float)K + p.D.eps);
  }
}
template <int NBT>
__device__ __forceinline__ float pick(const float (&v)[NBT], int b) {
  float r = v[0];
#pragma unroll
  for (int i = 1; i < NBT; ++i)
    if (i == b) r = v[i];
  return r;
}

// End of the LM-head instruction: combine the lanes' and warps' running argmax,
// publish this SM's best per lane; the last SM to arrive reduces all of them
// into the greedy ids and releases the step counter.
template <int NBT>
struct LmBest {  // running argmax per lane (value, index); passed by value, so it stays in registers
  float v[NBT];
  int i[NBT];
};
// the step's greedy keys, one per lane, at lmkey_off in the activation set
__device__ __forceinline__ unsigned long long* lm_keys(const KParams& p, const Misc* misc) {
  return reinterpret_cast<unsigned long long*>(misc->actset + p.lmkey_off);
}

template <int NBT>
static __device__ __noinline__ void lm_finish(const KParams& p, Misc* misc, const LmBest<NBT> best) {
  const Dims& D = p.D;
  const int ct = threadIdx.x - 32, cw = ct >> 5, lane = ct & 31;
#pragma unroll
  for (int b = 0; b < NBT; ++b) {
    float bv = best.v[b];
    int bi = best.i[b];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
      const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
      if (lm_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
    if (lane == 0) { misc->lmv[cw][b] = bv; misc->lmi[cw][b] = bi; }
  }
  cbar();
  if (ct < NBT) {
    float bv = -CUDART_INF_F;
    int bi = 0x7FFFFFFF;
    for (int w = 0; w < kConsumerWarps; ++w)
      if (lm_better(misc->lmv[w][ct], misc->lmi[w][ct], bv, bi)) { bv = misc->lmv[w][ct]; bi = misc->lmi[w][ct]; }
    // this SM's best joins the step's maximum (zeroed with the activation set)
    if (ct < p.nb && bi != 0x7FFFFFFF) atomicMax(lm_keys(p, misc) + ct, lm_key(bv, bi));
  }
  cbar();
  if (ct == 0) {
    const uint32_t old = atom_acq_rel_add(p.ctr + ctr_lm(D), 1u);
    misc->last = (old == gridDim.x - 1) && !misc->stop;
  }
  cbar();
  if (misc->last) {
    if (ct < p.nb) {  // every SM's maximum is in (ordered by the counter's acquire)
      const int bi = lm_key_row(ld_relaxed_u64(lm_keys(p, misc) + ct));
      p.ids[(size_t)misc->step * p.ids_stride + ct] = (bi >= 0 && bi < D.V) ? bi : 0;
    }
    cbar();
    if (ct == 0) {
      p.ctr[ctr_lm(D)] = 0u;                     // the next step's arrivals count from zero
      red_release_add(p.ctr + ctr_step(D), 1u);  // this step's ids are written
    }
  }
}

// Warp-per-page matvec over this instruction's units, then the op's epilogue.
// For QKV and GU the reduce-scatter keeps value pairs (rows j and j + RT/2 of a
// unit, same lane) in one lane: a RoPE pair for QKV, (gate, up) for GU; the
// other ops keep single values.
// Inlined into the consumer for 1-2 lanes: a call spills and reloads the
// caller's live registers for all 256 threads at every phase start (measured
// ~0.25 us); with 4-8 lanes the inlined accumulators would not fit the
// register budget, so those instantiations stay a call (mv_units_call).
template <int OPK, int RT, int NBT>
__device__ __forceinline__ void mv_units(const KParams& p, const Instr& I, uint32_t page_base,
                                      uint8_t* ring, const float* act, int K, uint64_t* full,
                                      uint64_t* empty, Misc* misc, uint32_t ii) {
  const Dims& D = p.D;
  constexpr int op = OPK;
  const int ct = threadIdx.x - 32, cw = ct >> 5, lane = ct & 31;
  const uint32_t NP = (uint32_t)p.ring_pages;
  const int nch = K >> 3;
  const uint32_t alo = smem_u32(act);
  const uint32_t ahi = alo + (uint32_t)(NBT * nch) * 16u;
  constexpr bool PL2 = OPK == OP_QKV || OPK == OP_GU;  // paired layout (RT >= 2 for these ops)
  constexpr int P = PL2 ? RT / 2 : 1;  // rows between the two values of a pair
  constexpr int NV = RT * NBT;
  constexpr int KEEP = PL2 ? 2 : 1;
  constexpr int NL = rs_left(NV, KEEP);
  const int vbase = rs_base(NV, KEEP, lane);
  const bool writer = (lane & rs_dup_mask(NV, KEEP)) == 0;
  // value m of this lane after the reduction: unit row vrow[m], lane vlane[m]
  int vrow[NL], vlane[NL];
#pragma unroll
  for (int m = 0; m < NL; ++m) {
    if (PL2) {
      const int pi = vbase / 2 + m / 2;
      vrow[m] = pi / NBT + (m & 1) * P;
      vlane[m] = pi % NBT;
    } else {
      vrow[m] = (vbase + m) / NBT;
      vlane[m] = (vbase + m) % NBT;
    }
  }
  LmBest<NBT> best;
#pragma unroll
  for (int b = 0; b < NBT; ++b) { best.v[b] = -CUDART_INF_F; best.i[b] = 0x7FFFFFFF; }
  long long* prec = p.prof ? p.prof + ((size_t)blockIdx.x * p.prof_stride + (ii - misc->i0)) * kProfSlots : nullptr;
  if (p.prof && lane == 0) { misc->warp_entry[cw] = (long long)globaltimer_ns(); misc->warp_first[cw] = 0; }
  float* lay = misc->actset + (size_t)I.layer * p.layer_floats;  // this layer's activation block
  // RMSNorm ops: the 1/rms scale of every value this lane holds after the reduction
  constexpr bool normed = op == OP_QKV || op == OP_GU || op == OP_LM;
  float osc[NL];
  if constexpr (normed) {
    float rinv[NBT];
    norm_scales<NBT>(p, misc, K, rinv);
#pragma unroll
    for (int m = 0; m < NL; ++m) osc[m] = pick<NBT>(rinv, vlane[m]);
  }
  long long c_wait = 0, c_pages = 0, c_core = 0, c_epi = 0;
  // this step's logits (LM head only)
  float* lg = nullptr;
  if (OPK == OP_LM && p.logits) {
    if (!p.logits_last) lg = p.logits + (size_t)misc->step * p.nb * D.V;
    else if (misc->step == p.n_steps - 1) lg = p.logits;
  }
  unsigned long long* accl = (OPK == OP_O || OPK == OP_DOWN) ? const_cast<unsigned long long*>(acc_of(p, misc, I.layer)) : nullptr;

  // a dynamic tail (gate/up, down, LM head): the units come with the pages, and
  // the stream position where the instruction ends is published by the producer
  constexpr bool DYN = OPK == OP_GU || OPK == OP_DOWN || OPK == OP_LM;
  const bool dyn = DYN && I.pool != 0;
  const uint32_t seq = (uint32_t)misc->step * misc->n_instr + (ii - misc->i0);
  RingPos rp;
  rp.init(page_base + cw, NP);
  for (uint32_t k = cw; dyn || k < I.n_units; k += kConsumerWarps, rp.advance(kConsumerWarps, NP)) {
    uint32_t u = I.u0 + k;
    const uint32_t slot = rp.slot;
    ResidIn rin[OPK == OP_O ? NL : 1];
    if constexpr (OPK == OP_O) {  // the residual rows this lane will write, loaded under the page wait
      const int r0 = (int)u * RT, nr = min(RT, D.H - r0);
#pragma unroll
      for (int m = 0; m < NL; ++m)
        if (writer && vrow[m] < nr && vlane[m] < p.nb) resid_issue(p, misc, I.layer, vlane[m], r0 + vrow[m], rin[m]);
    }
    const long long tw = prec ? (long long)globaltimer_ns() : 0;
    bool ok;
    if (DYN && dyn) {
      const int r = wait_dyn(p, &full[rp.fidx], rp.fphase, misc, seq, page_base + k, ii);
      if (__any_sync(0xFFFFFFFFu, r == 0)) break;  // every lane sees the same end
      ok = r > 0;
      if (ok) u = misc->unit[slot];
    } else {
      ok = wait_mbar(p, &full[rp.fidx], rp.fphase, E_WAIT_FULL, ii, true);
    }
    if (prec) {
      const long long now = (long long)globaltimer_ns();
      c_wait += now - tw;
      c_pages += 1;
      if (lane == 0 && misc->warp_first[cw] == 0) misc->warp_first[cw] = now;
    }
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) misc->stop = 1;
      break;
    }
    float2 acc[RT][NBT];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int b = 0; b < NBT; ++b) acc[r][b] = make_float2(0.f, 0.f);
    const long long tc = prec ? (long long)globaltimer_ns() : 0;
    mv_core<RT, NBT>(smem_u32(ring + (size_t)slot * kPageBytes), alo, ahi, nch, lane, acc);
    __syncwarp();
    if (lane == 0) mbar_arrive_cnt(&empty[slot], kConsumerWarps);
    const long long te = prec ? (long long)globaltimer_ns() : 0;
    if (prec) c_core += te - tc;

    float v[NV];
    if constexpr (PL2) {
#pragma unroll
      for (int j = 0; j < P; ++j)
#pragma unroll
        for (int b = 0; b < NBT; ++b)
#pragma unroll
          for (int h = 0; h < 2; ++h) v[(j * NBT + b) * 2 + h] = acc[j + h * P][b].x + acc[j + h * P][b].y;
    } else {
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int b = 0; b < NBT; ++b) v[r * NBT + b] = acc[r][b].x + acc[r][b].y;
    }
    warp_rs<NV, NV, KEEP, 16>(v, lane);
    if constexpr (normed) {
#pragma unroll
      for (int m = 0; m < NL; ++m) v[m] *= osc[m];
    }

    if constexpr (OPK == OP_QKV) {
      if constexpr (PL2) {
        const int half = D.d / 2;
        const int P0 = (int)u * P, hg = P0 / half, i0 = P0 % half;
        const int sec = hg < D.Hq ? 0 : (hg < D.Hq + D.Hkv ? 1 : 2);
        const int hh = sec == 0 ? hg : (sec == 1 ? hg - D.Hq : hg - D.Hq - D.Hkv);
#pragma unroll
        for (int m = 0; m < NL; m += 2) {
          const int b = vlane[m];
          if (!writer || b >= p.nb) continue;
          const float v1 = v[m], v2 = v[m + 1];
          const int i = i0 + vrow[m], pos = misc->pos[b];
          float r1 = v1, r2 = v2;
          if (sec < 2) {
            const float2 cs = misc->rope_cs[b][i];
            r1 = v1 * cs.x - v2 * cs.y;
            r2 = v2 * cs.x + v1 * cs.y;
          }
          if (sec == 0) {
            float* qq = lay + p.off_q + (size_t)b * D.qdim + hh * D.d;
            st_relaxed_f32(qq + i, canon(r1));
            st_relaxed_f32(qq + i + half, canon(r2));
          } else {
            // the cache row serves later steps; this step's attention reads the fp32 copy
            const size_t idx = ((((size_t)I.layer * D.n_phys_pages + misc->cur_phys[b]) * D.Hkv + hh) * 2 +
                                (sec - 1)) * (size_t)(D.PL * D.d) + (size_t)(pos % D.PL) * D.d + i;
            p.kv[idx] = D.kv_fp16 ? f2h(r1) : f2bf(r1);
            p.kv[idx + half] = D.kv_fp16 ? f2h(r2) : f2bf(r2);
            float* kv = lay + p.off_kvn + (size_t)b * 2 * D.kvdim + (sec - 1) * D.kvdim + hh * D.d;
            st_relaxed_f32(kv + i, canon(r1));
            st_relaxed_f32(kv + i + half, canon(r2));
          }
        }
      }
    } else if constexpr (OPK == OP_GU) {
      if constexpr (PL2) {
        const int r0 = (int)u * P, nr = min(P, D.F - r0);
#pragma unroll
        for (int m = 0; m < NL; m += 2) {
          const int r = vrow[m], b = vlane[m];
          if (!writer || r >= nr || b >= p.nb) continue;
          const float g = v[m], up = v[m + 1];
          st_relaxed_f32(lay + p.off_a + (size_t)b * D.F + r0 + r, canon(g / (1.0f + __expf(-g)) * up));
        }
      }
    } else if constexpr (OPK == OP_O) {  // x1 = residual + Wo . o, and x1 is the layer accumulator's first term
      const int r0 = (int)u * RT, nr = min(RT, D.H - r0);
#pragma unroll
      for (int m = 0; m < NL; ++m) {
        const int r = vrow[m], b = vlane[m];
        if (writer && r < nr && b < p.nb) {
          const float x1 = canon(resid_finish(p, misc, rin[m], ii) + v[m]);
          st_relaxed_f32(lay + p.off_x1 + (size_t)b * D.H + r0 + r, x1);
          red_acc(accl + (size_t)b * D.H + r0 + r, acc_enc(x1));
        }
      }
    } else if constexpr (OPK == OP_DOWN) {  // this K slice's term of the layer's residual
      const int r0 = (int)u * RT, nr = min(RT, D.H - r0);
#pragma unroll
      for (int m = 0; m < NL; ++m) {
        const int r = vrow[m], b = vlane[m];
        if (writer && r < nr && b < p.nb) red_acc(accl + (size_t)b * D.H + r0 + r, acc_enc(v[m]));
      }
    } else {  // OP_LM
      static_assert(OPK == OP_LM, "matvec op");
      const int r0 = (int)u * RT, nr = min(RT, D.V - r0);
#pragma unroll
      for (int m = 0; m < NL; ++m) {
        const int r = vrow[m], b = vlane[m];
        if (r >= nr || b >= p.nb) continue;
#pragma unroll
        for (int bb = 0; bb < NBT; ++bb)
          if (bb == b && lm_better(v[m], r0 + r, best.v[bb], best.i[bb])) { best.v[bb] = v[m]; best.i[bb] = r0 + r; }
        if (writer && lg) lg[(size_t)b * D.V + r0 + r] = v[m];
      }
    }
    if (prec) c_epi += (long long)globaltimer_ns() - te;
  }

  if (prec && lane == 0) {  // summed over the warps
    unsigned long long* pr = reinterpret_cast<unsigned long long*>(prec);
    atomicAdd(pr + 7, (unsigned long long)c_wait);
    atomicAdd(pr + 8, (unsigned long long)c_pages);
    atomicAdd(pr + 14, (unsigned long long)c_core);
    atomicAdd(pr + 15, (unsigned long long)c_epi);
  }
  if (p.prof && lane == 0) misc->warp_done[cw] = (long long)globaltimer_ns();  // profile only
  // this warp's share is written: bump the hint counter (every warp, pages or not)
  __syncwarp();
  if (lane == 0 && I.sig != kNoCounter) red_relaxed_add(p.ctr + I.sig, 1u);
  if constexpr (OPK == OP_LM) lm_finish<NBT>(p, misc, best);
}

// ---------------------------------------------------------------- consumers: tensor-core units

// Gate/up (OP_GU_TC) or the LM head (OP_LM_TC) of the 8-lane kernel on the
// tcgen05 tensor cores: a unit is a 128-row block of the weights over the whole
// K, streamed as nkt ring pages of 128 rows x 64 (16 KiB, pre-swizzled when the
// handle was created).  The staged activation is the B operand (stage<..., BOP>):
// 8 lanes' bf16 high parts then their low parts, N = 16, so the fp32 accumulator
// D[row][b] + D[row][8 + b] keeps the activations' fp32-level accuracy.  Consumer
// warp 0, lane 0 issues the MMAs (M = 128, N = 16, K = 16; four per page) into one
// of two accumulator buffers in tensor memory and releases each page's ring slot
// by committing to its empty barrier (it completes when the MMAs have read the
// page, without the issuer waiting for them).  A buffer is kTcAcc 16-column
// accumulators: MMA j of page kt adds into accumulator (kt & 1) * 4 + j, so
// consecutive MMAs never wait for one another's result (one accumulator for the
// whole K chains them: each waits out the previous one's latency, ~0.55 us per
// page measured).  Warps 4-7 (lane quarters 0-3 of tensor memory, one block row
// per thread) read a buffer back, sum its accumulators, scale by the lanes'
// 1/rms and run the epilogue: for
// gate/up, whose block rows alternate gate and up rows of the same ffn index, the
// two values meet by one shuffle and the even lane writes silu(g) * u; for the LM
// head, logits and the running argmax.  tc_n counts the units of every
// tensor-core instruction so far in this launch (the accumulator barriers'
// parities).  Measured faster than the CUDA cores with 8 lanes, where the CUDA-core
// matvec reads 32 bytes of activations from shared memory per 16 bytes of weights.
constexpr int kTcAcc = 8;                      // 16-column accumulators per buffer
constexpr uint32_t kTcCols = 2 * kTcAcc * 16;  // tensor-memory columns: two buffers
template <int OPK>
static __device__ __noinline__ void mv_units_tc(const KParams& p, const Instr& I, uint32_t page_base, uint8_t* ring,
                                                const float* act, uint64_t* full, uint64_t* empty, Misc* misc,
                                                uint32_t ii, uint32_t& tc_n) {
  constexpr int NBT = 8;
  static_assert(OPK == OP_GU_TC || OPK == OP_LM_TC, "tensor-core op");
  const Dims& D = p.D;
  const int ct = threadIdx.x - 32, lane = ct & 31;
  const int warp = threadIdx.x >> 5;  // 1..8; warp w reads tensor-memory lanes 32 (w % 4) ..
  const uint32_t NP = (uint32_t)p.ring_pages;
  const int nkt = D.nkt;
  const uint32_t tmem = misc->tmem_base;
  const uint32_t bsm = smem_u32(act);
  constexpr uint32_t kIdesc = idesc_bf16(128, 16);
  const int na = nkt >= 2 ? kTcAcc : kTcAcc / 2;  // accumulators a unit writes (pages 0 and 1 start them)
  float rinv[NBT];
  norm_scales<NBT>(p, misc, D.H, rinv);
  float* lay = misc->actset + (size_t)I.layer * p.layer_floats;
  float* lg = nullptr;
  if (OPK == OP_LM_TC && p.logits) {
    if (!p.logits_last) lg = p.logits + (size_t)misc->step * p.nb * D.V;
    else if (misc->step == p.n_steps - 1) lg = p.logits;
  }
  LmBest<NBT> best;
#pragma unroll
  for (int b = 0; b < NBT; ++b) { best.v[b] = -CUDART_INF_F; best.i[b] = 0x7FFFFFFF; }

  // profile mode: the issuer's page waits (and the epilogue's time, per unit)
  long long* prec = p.prof ? p.prof + ((size_t)blockIdx.x * p.prof_stride + (ii - misc->i0)) * kProfSlots : nullptr;
  long long c_wait = 0, c_pages = 0, c_epi = 0;
  if (warp == 1) {
    if (lane == 0) {  // the MMA issuer
      if (prec) { misc->warp_entry[0] = (long long)globaltimer_ns(); misc->warp_first[0] = 0; }
      RingPos rp;
      rp.init(page_base, NP);
      bool ok = true;
      for (uint32_t k = 0; k < I.n_units; ++k) {
        const uint32_t n = tc_n + k, buf = n & 1u;
        // the epilogue has read this accumulator's previous unit
        if (ok) ok = wait_mbar(p, &misc->tc_acce[buf], ((n >> 1) & 1u) ^ 1u, E_WAIT_FULL, ii, true);
        tc_fence_after();
        for (int kt = 0; kt < nkt; ++kt, rp.advance(1, NP)) {
          const long long tw = prec ? (long long)globaltimer_ns() : 0;
          if (ok) ok = wait_mbar(p, &full[rp.fidx], rp.fphase, E_WAIT_FULL, ii, true);
          if (prec) {
            const long long now = (long long)globaltimer_ns();
            c_wait += now - tw;
            c_pages += 1;
            if (misc->warp_first[0] == 0) misc->warp_first[0] = now;
          }
          if (ok) {
            tc_fence_after();
            const uint32_t a = smem_u32(ring + (size_t)rp.slot * kPageBytes), bb = bsm + (uint32_t)kt * 2048u;
            const uint32_t d = tmem + buf * (uint32_t)(kTcAcc * 16) + (uint32_t)(kt & 1) * 64u;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              umma_f16(d + 16u * j, sw128_desc(a + 32u * j), sw128_desc(bb + 32u * j), kIdesc, kt >= 2 ? 1u : 0u);
          }
          // the slot is free once these MMAs have read the page: the barrier counts
          // the 8 arrivals a consumer page release gives; 7 now, and the last from a
          // commit, when every MMA issued so far has completed
          mbar_arrive_cnt(&empty[rp.slot], (uint32_t)kConsumerWarps - 1u);
          umma_commit(&empty[rp.slot]);
        }
        umma_commit(&misc->tc_accf[buf]);  // the unit's accumulator is complete
      }
    }
  } else if (warp >= 4) {
    if (warp <= 7) {  // the epilogue: tensor-memory lane quarter warp % 4
      const int qd = warp & 3;
      for (uint32_t k = 0; k < I.n_units; ++k) {
        const uint32_t n = tc_n + k, buf = n & 1u;
        const bool ok =
            __all_sync(0xFFFFFFFFu, wait_mbar(p, &misc->tc_accf[buf], (n >> 1) & 1u, E_WAIT_FULL, ii, true));
        const long long te = prec ? (long long)globaltimer_ns() : 0;
        tc_fence_after();
        float v[NBT];
#pragma unroll
        for (int b = 0; b < NBT; ++b) v[b] = 0.f;
        const uint32_t ta = tmem + ((uint32_t)(32 * qd) << 16) + buf * (uint32_t)(kTcAcc * 16);
        for (int a = 0; a < na; a += 2) {  // two accumulators per load
          uint32_t r[32];
          tmem_ld32(ta + 16u * (uint32_t)a, r);
          tmem_ld_wait();
#pragma unroll
          for (int b = 0; b < NBT; ++b)
            v[b] += (__uint_as_float(r[b]) + __uint_as_float(r[8 + b])) +
                    (__uint_as_float(r[16 + b]) + __uint_as_float(r[24 + b]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&misc->tc_acce[buf]);
        if (!ok) continue;
#pragma unroll
        for (int b = 0; b < NBT; ++b) v[b] *= rinv[b];
        const int u = (int)(I.u0 + k);
        if constexpr (OPK == OP_GU_TC) {
          const int row = 32 * qd + lane, f = 64 * u + (row >> 1);  // even rows gate, odd rows up
#pragma unroll
          for (int b = 0; b < NBT; ++b) {
            const float up = __shfl_xor_sync(0xFFFFFFFFu, v[b], 1);
            if (!(lane & 1) && b < p.nb && f < D.F)
              st_relaxed_f32(lay + p.off_a + (size_t)b * D.F + f, canon(v[b] / (1.0f + __expf(-v[b])) * up));
          }
        } else {
          const int row = 128 * u + 32 * qd + lane;
          if (row < D.V) {
#pragma unroll
            for (int b = 0; b < NBT; ++b) {
              if (b >= p.nb) break;
              if (lm_better(v[b], row, best.v[b], best.i[b])) { best.v[b] = v[b]; best.i[b] = row; }
              if (lg) lg[(size_t)b * D.V + row] = v[b];
            }
          }
        }
        if (prec) c_epi += (long long)globaltimer_ns() - te;
      }
    }
  }
  if (prec && lane == 0 && (c_pages || c_epi)) {  // summed over the warps, like the matvec's
    unsigned long long* pr = reinterpret_cast<unsigned long long*>(prec);
    atomicAdd(pr + 7, (unsigned long long)c_wait);
    atomicAdd(pr + 8, (unsigned long long)c_pages);
    atomicAdd(pr + 15, (unsigned long long)c_epi);
  }
  tc_n += I.n_units;
  // this warp's share is written: bump the hint counter (every warp, as the matvec does)
  __syncwarp();
  if (lane == 0 && I.sig != kNoCounter) red_relaxed_add(p.ctr + I.sig, 1u);
  if constexpr (OPK == OP_LM_TC) lm_finish<NBT>(p, misc, best);
}

// ---------------------------------------------------------------- consumers: attention

// The last slice of a (lane, kv head) with many slices merges them: their (m, l)
// go to shared memory once (comb is free: the slice's own states are in its
// partial), each head's weights exp(m_t - M) / L are computed once, and the outputs
// are summed with batches of independent loads, so the merge costs a few L2 round
// trips instead of three per slice.  Compiled into the 128-dim-head kernels only
// (8B batch 1, 2048-token context: 2909.7 -> 2739.3 us/step).  In the 64-dim
// kernels it measured 1B 8192-token context 644.8 -> 626.6 but batch 4 919.6 ->
// 939.0 and batch 1 +0.6 to +3.6, inline or out of line, from the larger attention
// code alone (those merges were not executed); they keep the per-thread walk.
template <int DH, int REP>
__device__ __forceinline__ void merge_slices_staged(const KParams& p, const Instr& I, float* comb, float* lay,
                                                        int b, int g, int se) {
  constexpr int CS = DH + 2;
  const Dims& D = p.D;
  const int ct = threadIdx.x - 32;
  const float* pp = p.part + (size_t)(b * D.Hkv + g) * p.S * REP * CS;
  float* sm_m = comb;              // [se][REP] maxima
  float* sm_l = comb + se * REP;   // [se][REP] sums, then the weights
  for (int e = ct; e < se * REP; e += 256) {
    const float* rec = pp + e * CS;  // record (t, h) = e: slice t = e / REP, head h = e % REP
    sm_m[e] = __ldcg(rec + DH);
    sm_l[e] = __ldcg(rec + DH + 1);
  }
  cbar();
  if (ct < REP) {
    float M = -CUDART_INF_F;
    for (int t = 0; t < se; ++t) M = fmaxf(M, sm_m[t * REP + ct]);
    float L = 0.f;
    for (int t = 0; t < se; ++t) {
      const float mt = sm_m[t * REP + ct];
      if (mt > -CUDART_INF_F) L += sm_l[t * REP + ct] * __expf(mt - M);
    }
    const float invL = 1.0f / L;
    for (int t = 0; t < se; ++t) {
      const float mt = sm_m[t * REP + ct];
      sm_l[t * REP + ct] = mt > -CUDART_INF_F ? __expf(mt - M) * invL : 0.f;
    }
  }
  cbar();
  for (int e = ct; e < REP * DH; e += 256) {
    const int h = e / DH, i = e % DH;
    const float* src = pp + h * CS + i;  // slice t's value at src + t * REP * CS
    float O = 0.f;
    int t = 0;
    for (; t + 6 <= se; t += 6) {
      float v[6];
#pragma unroll
      for (int k = 0; k < 6; ++k) v[k] = __ldcg(src + (size_t)(t + k) * REP * CS);
#pragma unroll
      for (int k = 0; k < 6; ++k) O = fmaf(v[k], sm_l[(t + k) * REP + h], O);
    }
    for (; t < se; ++t) O = fmaf(__ldcg(src + (size_t)t * REP * CS), sm_l[t * REP + h], O);
    st_relaxed_f32(lay + p.off_o + (size_t)b * D.qdim + (g * REP + h) * DH + i, canon(O));
  }
  cbar();
  if (ct == 0) {
    p.ctr[ctr_part(D, I.layer, b, g)] = 0u;  // the next step's slices count from zero
    red_relaxed_add(p.ctr + ctr_layer(I.layer, C_ATTN), 1u);
  }
}

// Slices per (lane, kv head) from which the last slice merges through shared memory.
constexpr int kMergeStaged = 8;

// Split-KV GQA decode attention of one slice: the REP query heads of kv head g
// over KV pages [pb, pe) of lane b's context (npg pages).  The pages are dealt to
// the 8 warps like matvec pages (warp w takes the slice's pages w, w + 8, ...),
// and each warp folds its pages into an online-softmax state of its own (running
// max m, sum l, unnormalised o per query head): per page, a lane scores its
// PL / 32 positions against every head, the warp reduces each head's maximum and
// sum, writes the probabilities to its own shared-memory rows, and P V runs with
// a lane per DH / 32 output dims.  Warps work on different pages at the same
// time, so a slice of n pages costs about n / 8 page latencies, not n.  After the
// slice the CTA merges the 8 warp states into the slice's partial; a slice that
// covers all pages writes o directly, otherwise the last slice to finish (atomic
// counter) merges all slices of the (lane, kv head) into o.  This step's K/V row
// comes from the fp32 copy the QKV instruction published, rounded as the cache
// holds it, and is patched into the last page by the warp that owns that page.
// Returns false when the CTA stopped.
template <int DH, int REP, bool KV16F>
__device__ __forceinline__ bool attn_one(const KParams& p, const Instr& I, uint32_t page_base, uint8_t* ring,
                                         float* act, uint64_t* full, uint64_t* empty, Misc* misc, uint32_t ii,
                                         int b, int g, int pb, int pe, int npg, int s, int se) {
  constexpr int DC = DH / 8;                 // 16-byte chunks per K/V row
  constexpr int PL = kPageBytes / (4 * DH);  // positions per KV page
  constexpr int TPL = PL / 32;               // positions per lane in a page
  constexpr int DPL = DH / 32;               // output dims per lane
  constexpr int CS = DH + 2;                 // partial record: o[DH], m, l
  static_assert(PL % 32 == 0, "positions per page");
  static_assert(kConsumerWarps * PL * REP <= kConsumerWarps * REP * CS, "probabilities alias the combine scratch");
  const Dims& D = p.D;
  const int ct = threadIdx.x - 32, cw = ct >> 5, lane = ct & 31;
  const uint32_t NP = (uint32_t)p.ring_pages;
  float4* qlo = reinterpret_cast<float4*>(act);
  float4* qhi = qlo + REP * DC;
  const uint32_t sqlo = smem_u32(qlo), sqhi = smem_u32(qhi);
  float* comb = act + REP * DH;
  float* pw = comb + cw * PL * REP;  // this warp's probabilities [PL][REP] (aliases comb until the merge)
  const float scale = 1.0f / sqrtf((float)DH);
  float* lay = misc->actset + (size_t)I.layer * p.layer_floats;
  const int pos = misc->pos[b];
  const int np_ = pe - pb;
  // the warp that owns the slice's last page patches this step's K/V row into it
  const bool own_cur = pe == npg && (np_ - 1) % kConsumerWarps == cw;
  const int rcur = pos - (npg - 1) * PL;
  uint32_t kcur[DH / 64], vcur[DH / 64];
  if (own_cur) {
    const float* kn = lay + p.off_kvn + (size_t)b * 2 * D.kvdim + g * DH + lane * (DH / 32);
    const float* vn = kn + D.kvdim;
    float kf[DH / 32], vf[DH / 32];
    if constexpr (DH == 64) {
      float2 k2 = ld_relaxed_f2(kn), v2 = ld_relaxed_f2(vn);
      ready(k2, p, kn, ii, misc);
      ready(v2, p, vn, ii, misc);
      kf[0] = k2.x; kf[1] = k2.y; vf[0] = v2.x; vf[1] = v2.y;
    } else {
      float4 k4 = ld_relaxed_f4(kn), v4 = ld_relaxed_f4(vn);
      ready(k4, p, kn, ii, misc);
      ready(v4, p, vn, ii, misc);
      kf[0] = k4.x; kf[1] = k4.y; kf[2] = k4.z; kf[3] = k4.w;
      vf[0] = v4.x; vf[1] = v4.y; vf[2] = v4.z; vf[3] = v4.w;
    }
#pragma unroll
    for (int e = 0; e < DH / 64; ++e) {
      kcur[e] = KV16F ? (uint32_t)f2h(kf[2 * e]) | ((uint32_t)f2h(kf[2 * e + 1]) << 16)
                      : (uint32_t)f2bf(kf[2 * e]) | ((uint32_t)f2bf(kf[2 * e + 1]) << 16);
      vcur[e] = KV16F ? (uint32_t)f2h(vf[2 * e]) | ((uint32_t)f2h(vf[2 * e + 1]) << 16)
                      : (uint32_t)f2bf(vf[2 * e]) | ((uint32_t)f2bf(vf[2 * e + 1]) << 16);
    }
  }
  for (int e = ct; e < REP * DC; e += 256) {
    const int h = e / DC, c = e % DC;
    const float* src = lay + p.off_q + (size_t)b * D.qdim + (g * REP + h) * DH + c * 8;
    float4 a0 = ld_relaxed_f4(src), a1 = ld_relaxed_f4(src + 4);
    ready(a0, p, src, ii, misc);
    ready(a1, p, src + 4, ii, misc);
    a0.x *= scale; a0.y *= scale; a0.z *= scale; a0.w *= scale;
    a1.x *= scale; a1.y *= scale; a1.z *= scale; a1.w *= scale;
    qlo[h * DC + c] = a0;
    qhi[h * DC + c] = a1;
  }
  cbar();

  float m[REP], l[REP], o[REP][DPL];
#pragma unroll
  for (int h = 0; h < REP; ++h) {
    m[h] = -CUDART_INF_F;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) o[h][e] = 0.f;
  }
  RingPos rp;
  rp.init(page_base + cw, NP);
  for (int j = cw; j < np_; j += kConsumerWarps, rp.advance(kConsumerWarps, NP)) {
    const uint32_t slot = rp.slot;
    const bool ok = wait_mbar(p, &full[rp.fidx], rp.fphase, E_WAIT_FULL, ii, true);
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) misc->stop = 1;
      break;
    }
    uint8_t* pg = ring + (size_t)slot * kPageBytes;
    uint8_t* vpg = pg + PL * DH * 2;
    const int cnt = min(PL, pos + 1 - (pb + j) * PL);  // positions of this page up to pos, >= 1
    const bool patch = own_cur && j == np_ - 1;
    if (patch) {  // this step's K/V, written by the QKV instruction, replace the stale copy
#pragma unroll
      for (int e = 0; e < DH / 64; ++e) {
        reinterpret_cast<uint32_t*>(pg + rcur * DH * 2)[lane * (DH / 64) + e] = kcur[e];
        reinterpret_cast<uint32_t*>(vpg + rcur * DH * 2)[lane * (DH / 64) + e] = vcur[e];
      }
      __syncwarp();
    }
    // scores: position lane + 32 t against every head
    float2 a2[TPL][REP];
#pragma unroll
    for (int t = 0; t < TPL; ++t)
#pragma unroll
      for (int h = 0; h < REP; ++h) a2[t][h] = make_float2(0.f, 0.f);
    const uint32_t kb = smem_u32(pg);
#pragma unroll 2
    for (int cc = 0; cc < DC; ++cc) {
      const int c = (cc + lane) & (DC - 1);  // lanes of a phase hit distinct banks
      uint4 kw[TPL];
#pragma unroll
      for (int t = 0; t < TPL; ++t) kw[t] = lds128(kb + (uint32_t)(((lane + 32 * t) * DC + c) * 16));
#pragma unroll
      for (int h = 0; h < REP; ++h) {
        const float4 ql = lds128f(sqlo + (uint32_t)((h * DC + c) * 16));
        const float4 qh = lds128f(sqhi + (uint32_t)((h * DC + c) * 16));
#pragma unroll
        for (int t = 0; t < TPL; ++t) {
          float2 acc = a2[t][h];
          acc = __ffma2_rn(make_float2(kv_lo<KV16F>(kw[t].x), kv_hi<KV16F>(kw[t].x)), make_float2(ql.x, ql.y), acc);
          acc = __ffma2_rn(make_float2(kv_lo<KV16F>(kw[t].y), kv_hi<KV16F>(kw[t].y)), make_float2(ql.z, ql.w), acc);
          acc = __ffma2_rn(make_float2(kv_lo<KV16F>(kw[t].z), kv_hi<KV16F>(kw[t].z)), make_float2(qh.x, qh.y), acc);
          acc = __ffma2_rn(make_float2(kv_lo<KV16F>(kw[t].w), kv_hi<KV16F>(kw[t].w)), make_float2(qh.z, qh.w), acc);
          a2[t][h] = acc;
        }
      }
    }
    // online softmax per head over this page's positions
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      float sc[TPL], mx = -CUDART_INF_F;
#pragma unroll
      for (int t = 0; t < TPL; ++t) {
        sc[t] = lane + 32 * t < cnt ? a2[t][h].x + a2[t][h].y : -CUDART_INF_F;
        mx = fmaxf(mx, sc[t]);
      }
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o2));
      const float mn = fmaxf(m[h], mx);  // finite: position 0 of every page is valid
      const float corr = __expf(m[h] - mn);
      float ps = 0.f;
#pragma unroll
      for (int t = 0; t < TPL; ++t) {
        const float pr = sc[t] > -CUDART_INF_F ? __expf(sc[t] - mn) : 0.f;
        pw[(lane + 32 * t) * REP + h] = pr;
        ps += pr;
      }
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) ps += __shfl_xor_sync(0xFFFFFFFFu, ps, o2);
      l[h] = l[h] * corr + ps;
      m[h] = mn;
#pragma unroll
      for (int e = 0; e < DPL; ++e) o[h][e] *= corr;
    }
    __syncwarp();
    // o[h][dims of this lane] += p[position][h] * v[position][dims]
    const uint32_t vb = smem_u32(vpg) + (uint32_t)(lane * DPL * 2);
#pragma unroll 4
    for (int r = 0; r < cnt; ++r) {
      float vv[DPL];
      if constexpr (DPL == 2) {
        const uint32_t w = lds32(vb + (uint32_t)(r * DH * 2));
        vv[0] = kv_lo<KV16F>(w); vv[1] = kv_hi<KV16F>(w);
      } else {
        const uint2 w = lds64(vb + (uint32_t)(r * DH * 2));
        vv[0] = kv_lo<KV16F>(w.x); vv[1] = kv_hi<KV16F>(w.x); vv[2] = kv_lo<KV16F>(w.y); vv[3] = kv_hi<KV16F>(w.y);
      }
      float ph[REP];
      if constexpr (REP % 4 == 0) {
#pragma unroll
        for (int h = 0; h < REP; h += 4) {
          const float4 p4 = *reinterpret_cast<const float4*>(pw + r * REP + h);
          ph[h] = p4.x; ph[h + 1] = p4.y; ph[h + 2] = p4.z; ph[h + 3] = p4.w;
        }
      } else {
#pragma unroll
        for (int h = 0; h < REP; ++h) ph[h] = pw[r * REP + h];
      }
#pragma unroll
      for (int h = 0; h < REP; ++h)
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[h][e] = fmaf(ph[h], vv[e], o[h][e]);
    }
    __syncwarp();
    if (patch) fence_proxy_async_smem();  // generic writes before the next bulk copy into the slot
    if (lane == 0) mbar_arrive_cnt(&empty[slot], kConsumerWarps);
  }
  cbar();  // every warp is done with its probabilities (they alias comb)
  // the warps' states into comb, then merged into this slice's partial
  float* mine = comb + cw * REP * CS;
#pragma unroll
  for (int h = 0; h < REP; ++h) {
#pragma unroll
    for (int e = 0; e < DPL; ++e) mine[h * CS + lane * DPL + e] = o[h][e];
    if (lane == 0) { mine[h * CS + DH] = m[h]; mine[h * CS + DH + 1] = l[h]; }
  }
  cbar();
  if (misc->stop) { cbar(); return false; }
  if (se == 1) {
    // the only slice of these heads: normalise and write the output, then signal
    for (int e = ct; e < REP * DH; e += 256) {
      const int h = e / DH, i = e % DH;
      float M = -CUDART_INF_F;
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, comb[(w * REP + h) * CS + DH]);
      float L = 0.f, O = 0.f;
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mw = comb[(w * REP + h) * CS + DH];
        if (mw > -CUDART_INF_F) {
          const float f = __expf(mw - M);
          L += comb[(w * REP + h) * CS + DH + 1] * f;
          O += comb[(w * REP + h) * CS + i] * f;
        }
      }
      st_relaxed_f32(lay + p.off_o + (size_t)b * D.qdim + (g * REP + h) * DH + i, canon(O / L));
    }
    cbar();
    if (ct == 0) red_relaxed_add(p.ctr + ctr_layer(I.layer, C_ATTN), 1u);
    cbar();
    return true;
  }
  float* part = p.part + ((size_t)(b * D.Hkv + g) * p.S + s) * REP * CS;
  for (int e = ct; e < REP * DH; e += 256) {
    const int h = e / DH, i = e % DH;
    float M = -CUDART_INF_F;
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, comb[(w * REP + h) * CS + DH]);
    float L = 0.f, O = 0.f;
    if (M > -CUDART_INF_F)
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mw = comb[(w * REP + h) * CS + DH];
        if (mw > -CUDART_INF_F) {
          const float f = __expf(mw - M);
          L += comb[(w * REP + h) * CS + DH + 1] * f;
          O += comb[(w * REP + h) * CS + i] * f;
        }
      }
    part[h * CS + i] = O;
    if (i == 0) { part[h * CS + DH] = M; part[h * CS + DH + 1] = L; }
  }
  cbar();
  if (ct == 0) {
    const uint32_t old = atom_acq_rel_add(p.ctr + ctr_part(D, I.layer, b, g), 1u);
    misc->last = (old == (uint32_t)se - 1);
  }
  cbar();
  if (misc->last && (DH < 128 || se < kMergeStaged)) {  // each thread walks the slices
    const float* pp = p.part + (size_t)(b * D.Hkv + g) * p.S * REP * CS;
    for (int e = ct; e < REP * DH; e += 256) {
      const int h = e / DH, i = e % DH;
      float M = -CUDART_INF_F;
      for (int t = 0; t < se; ++t) M = fmaxf(M, __ldcg(pp + (t * REP + h) * CS + DH));
      float L = 0.f, O = 0.f;
      for (int t = 0; t < se; ++t) {
        const float mt = __ldcg(pp + (t * REP + h) * CS + DH);
        if (mt > -CUDART_INF_F) {
          const float f = __expf(mt - M);
          L += __ldcg(pp + (t * REP + h) * CS + DH + 1) * f;
          O += __ldcg(pp + (t * REP + h) * CS + i) * f;
        }
      }
      st_relaxed_f32(lay + p.off_o + (size_t)b * D.qdim + (g * REP + h) * DH + i, canon(O / L));
    }
    cbar();
    if (ct == 0) {
      p.ctr[ctr_part(D, I.layer, b, g)] = 0u;  // the next step's slices count from zero
      red_relaxed_add(p.ctr + ctr_layer(I.layer, C_ATTN), 1u);
    }
  } else if constexpr (DH >= 128) {
    if (misc->last) merge_slices_staged<DH, REP>(p, I, comb, lay, b, g, se);
  }
  cbar();
  return true;
}

// Short-context attention of one query head (the head split of attn_plan):
// every position of lane b's context (npg <= kHeadSplitPages pages, at most 256
// positions) is scored at once, one position per thread, then a block-wide
// softmax, then P.V with one thread per (pair of output dims, run of 32
// positions within one page).  The
// pages of the unit are all resident in the ring (npg <= 4 <= ring pages).
template <int DH, bool KV16F>
__device__ __forceinline__ bool attn_flat(const KParams& p, const Instr& I, uint32_t page_base, uint8_t* ring,
                                          float* act, uint64_t* full, uint64_t* empty, Misc* misc, uint32_t ii,
                                          int b, int g, int hq, int npg) {
  constexpr int PL = kPageBytes / (4 * DH);  // positions per KV page
  constexpr int DC = DH / 8;                 // 16-byte chunks per K row
  constexpr int WPR = DH / 2;                       // 32-bit words (dim pairs) per V row
  constexpr int NCH = kConsumerWarps * 32 / WPR;   // runs of positions in P.V
  constexpr int RUN = kHeadSplitPages * PL / NCH;  // positions per run
  static_assert(kHeadSplitPages * PL <= kConsumerWarps * 32, "one position per thread");
  static_assert(PL % RUN == 0, "a run stays within one page");
  const Dims& D = p.D;
  const int ct = threadIdx.x - 32, cw = ct >> 5, lane = ct & 31;
  const uint32_t NP = (uint32_t)p.ring_pages;
  float* qs = act;            // [DH] query, scaled by 1/sqrt(d)
  float* ps = qs + DH;        // [256] unnormalised probabilities
  float* wred = ps + 256;     // [2][8] per-warp maxima, sums
  float* part = wred + 16;    // [NCH][DH] partial outputs (NCH * DH = 512)
  float* lay = misc->actset + (size_t)I.layer * p.layer_floats;
  const int pos = misc->pos[b], cnt = pos + 1;
  // ring slots of the unit's pages
  uint32_t slot[kHeadSplitPages];
  {
    RingPos rp;
    rp.init(page_base, NP);
#pragma unroll
    for (int j = 0; j < kHeadSplitPages; ++j, rp.advance(1, NP)) slot[j] = rp.slot;
  }
  // the query, and this step's K/V row patched into the last page (rounded as the
  // cache holds it; the page's bulk copy stops short of that row)
  if (ct < DH / 4) {
    const float* src = lay + p.off_q + (size_t)b * D.qdim + hq * DH + ct * 4;
    float4 v = ld_relaxed_f4(src);
    ready(v, p, src, ii, misc);
    const float sc = 1.0f / sqrtf((float)DH);
    reinterpret_cast<float4*>(qs)[ct] = make_float4(v.x * sc, v.y * sc, v.z * sc, v.w * sc);
  }
  const int rcur = pos - (npg - 1) * PL;
  uint8_t* lastpg = ring + (size_t)slot[npg - 1 < 0 ? 0 : npg - 1] * kPageBytes;
  const bool patcher = ct >= 32 && ct < 32 + DH / 2;  // warp 1 (and 2 for DH = 128)
  if (patcher) {
    const int e = ct - 32;  // element pair (2e, 2e + 1)
    const float* kn = lay + p.off_kvn + (size_t)b * 2 * D.kvdim + g * DH + 2 * e;
    float2 k2 = ld_relaxed_f2(kn), v2 = ld_relaxed_f2(kn + D.kvdim);
    ready(k2, p, kn, ii, misc);
    ready(v2, p, kn + D.kvdim, ii, misc);
    const uint32_t kw = KV16F ? (uint32_t)f2h(k2.x) | ((uint32_t)f2h(k2.y) << 16)
                              : (uint32_t)f2bf(k2.x) | ((uint32_t)f2bf(k2.y) << 16);
    const uint32_t vw = KV16F ? (uint32_t)f2h(v2.x) | ((uint32_t)f2h(v2.y) << 16)
                              : (uint32_t)f2bf(v2.x) | ((uint32_t)f2bf(v2.y) << 16);
    reinterpret_cast<uint32_t*>(lastpg + rcur * DH * 2)[e] = kw;
    reinterpret_cast<uint32_t*>(lastpg + PL * DH * 2 + rcur * DH * 2)[e] = vw;
  }
  // every warp waits for all pages (each warp releases each page once, below)
  bool ok = true;
  {
    RingPos rp;
    rp.init(page_base, NP);
    for (int j = 0; j < npg && ok; ++j, rp.advance(1, NP)) ok = wait_mbar(p, &full[rp.fidx], rp.fphase, E_WAIT_FULL, ii, true);
  }
  if (!__all_sync(0xFFFFFFFFu, ok) && lane == 0) misc->stop = 1;
  cbar();
  if (misc->stop) { cbar(); return false; }
  // scores: thread t -> position t
  float sv = -CUDART_INF_F;
  if (ct < cnt) {
    const int j = ct / PL, row = ct % PL;
    uint32_t sl = slot[0];
#pragma unroll
    for (int jj = 1; jj < kHeadSplitPages; ++jj)
      if (jj == j) sl = slot[jj];
    const uint32_t krow = smem_u32(ring + (size_t)sl * kPageBytes) + (uint32_t)(row * DH * 2);
    const uint32_t qa = smem_u32(qs);
    float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int cc = 0; cc < DC; ++cc) {
      const int c = (cc + lane) & (DC - 1);  // lanes of a phase hit distinct banks
      const uint4 kw = lds128(krow + (uint32_t)(c * 16));
      const float4 q0 = lds128f(qa + (uint32_t)(c * 32)), q1 = lds128f(qa + (uint32_t)(c * 32 + 16));
      a2 = __ffma2_rn(make_float2(kv_lo<KV16F>(kw.x), kv_hi<KV16F>(kw.x)), make_float2(q0.x, q0.y), a2);
      a2 = __ffma2_rn(make_float2(kv_lo<KV16F>(kw.y), kv_hi<KV16F>(kw.y)), make_float2(q0.z, q0.w), a2);
      a2 = __ffma2_rn(make_float2(kv_lo<KV16F>(kw.z), kv_hi<KV16F>(kw.z)), make_float2(q1.x, q1.y), a2);
      a2 = __ffma2_rn(make_float2(kv_lo<KV16F>(kw.w), kv_hi<KV16F>(kw.w)), make_float2(q1.z, q1.w), a2);
    }
    sv = a2.x + a2.y;
  }
  // block max, then probabilities and their sum
  float mx = sv;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if (lane == 0) wred[cw] = mx;
  cbar();
  float M = wred[0];
#pragma unroll
  for (int w = 1; w < kConsumerWarps; ++w) M = fmaxf(M, wred[w]);
  const float e = ct < cnt ? __expf(sv - M) : 0.f;
  ps[ct] = e;
  float sum = e;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  if (lane == 0) wred[8 + cw] = sum;
  cbar();
  // P.V: thread (word wd = dims 2wd, 2wd + 1; run ch) sums positions [ch * RUN, ch * RUN + RUN)
  {
    const int wd = ct % WPR, ch = ct / WPR;
    const int t0 = ch * RUN, t1 = min(cnt, t0 + RUN);
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
    if (t0 < t1) {
      const int j = t0 / PL;
      uint32_t sl = slot[0];
#pragma unroll
      for (int jj = 1; jj < kHeadSplitPages; ++jj)
        if (jj == j) sl = slot[jj];
      const uint32_t vb = smem_u32(ring + (size_t)sl * kPageBytes + PL * DH * 2) +
                          (uint32_t)((t0 % PL) * DH * 2 + wd * 4);
      const float* pp = ps + t0;
      const int n = t1 - t0;
      int t = 0;
#pragma unroll 4
      for (; t + 2 <= n; t += 2) {
        const uint32_t w0 = lds32(vb + (uint32_t)(t * DH * 2)), w1 = lds32(vb + (uint32_t)((t + 1) * DH * 2));
        const float p0 = pp[t], p1 = pp[t + 1];
        a0 = fmaf(p0, kv_lo<KV16F>(w0), a0);
        a1 = fmaf(p0, kv_hi<KV16F>(w0), a1);
        b0 = fmaf(p1, kv_lo<KV16F>(w1), b0);
        b1 = fmaf(p1, kv_hi<KV16F>(w1), b1);
      }
      if (t < n) {
        const uint32_t w0 = lds32(vb + (uint32_t)(t * DH * 2));
        a0 = fmaf(pp[t], kv_lo<KV16F>(w0), a0);
        a1 = fmaf(pp[t], kv_hi<KV16F>(w0), a1);
      }
    }
    part[ch * DH + 2 * wd] = a0 + b0;
    part[ch * DH + 2 * wd + 1] = a1 + b1;
  }
  // every read of the pages is done: release them (the patch first, to the async proxy)
  if (patcher) fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0)
    for (int j = 0; j < npg; ++j) mbar_arrive_cnt(&empty[slot[j]], 1u);
  cbar();
  if (ct < DH) {
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) L += wred[8 + w];
    float O = 0.f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) O += part[c * DH + ct];
    st_relaxed_f32(lay + p.off_o + (size_t)b * D.qdim + hq * DH + ct, canon(O / L));
  }
  cbar();
  if (ct == 0) red_relaxed_add(p.ctr + ctr_layer(I.layer, C_ATTN), 1u);
  return true;
}

// Split-KV GQA decode attention for the units of this instruction (see
// attn_plan): a slice covers a contiguous range of KV pages of one (lane, kv
// head) and all its query heads, or, for short contexts, one query head over
// all pages.  Every page is shared by the 8 warps, each taking PL/8 of its
// positions: a lane scores one (position, query head) pair, then each warp folds
// its positions into an online-softmax partial (running max m, sum l,
// unnormalised o).  After the slice the CTA combines the warps' partials; a
// slice that covers all pages writes o, otherwise the last slice to finish
// (atomic counter) merges all slices of the (lane, kv head) into o.  Returns the
// ring pages consumed.
template <int DH, int REP, bool KV16F>
__device__ __forceinline__ uint32_t attn_units_body(const KParams& p, const Instr& I, uint32_t page_base,
                                                    uint8_t* ring, float* act, uint64_t* full, uint64_t* empty,
                                                    Misc* misc, uint32_t ii) {
  constexpr int PL = kPageBytes / (4 * DH);
  const Dims& D = p.D;
  uint32_t used = 0;
  for (uint32_t k = 0; k < I.n_units; ++k) {
    int b, g, s;
    attn_unit(I.u0 + k, D.Hkv, p.S, &b, &g, &s);
    const int npg = misc->pos[b] / PL + 1;
    const AttnPlan ap = attn_plan(p.S, REP, npg, s);
    if (!ap.active) continue;  // uniform: this slice is not needed at this context length
    bool ok;
    if (REP > 1 && ap.single)
      ok = attn_flat<DH, KV16F>(p, I, page_base + used, ring, act, full, empty, misc, ii, b, g, g * REP + ap.head,
                                npg);
    else
      ok = attn_one<DH, REP, KV16F>(p, I, page_base + used, ring, act, full, empty, misc, ii, b, g, ap.pb, ap.pe,
                                    npg, s, ap.se);
    if (!ok) break;
    used += (uint32_t)(ap.pe - ap.pb);
  }
  return used;
}
template <int DH, int REP, bool KV16F>
static __device__ __noinline__ uint32_t attn_units(const KParams& p, const Instr& I, uint32_t page_base, uint8_t* ring,
                                            float* act, uint64_t* full, uint64_t* empty, Misc* misc, uint32_t ii) {
  return attn_units_body<DH, REP, KV16F>(p, I, page_base, ring, act, full, empty, misc, ii);
}

// ---------------------------------------------------------------- consumers: ops

template <int OPK, int RT, int NBT>
static __device__ __noinline__ void mv_units_call(const KParams& p, const Instr& I, uint32_t pb, uint8_t* ring,
                                           const float* act, int K, uint64_t* full, uint64_t* empty, Misc* misc,
                                           uint32_t ii) {
  mv_units<OPK, RT, NBT>(p, I, pb, ring, act, K, full, empty, misc, ii);
}
template <int OPK, int RT, int NBT>
__device__ __forceinline__ void mv_run(const KParams& p, const Instr& I, uint32_t pb, uint8_t* ring,
                                       const float* act, int K, uint64_t* full, uint64_t* empty, Misc* misc,
                                       uint32_t ii) {
  if constexpr (NBT <= 2) mv_units<OPK, RT, NBT>(p, I, pb, ring, act, K, full, empty, misc, ii);
  else mv_units_call<OPK, RT, NBT>(p, I, pb, ring, act, K, full, empty, misc, ii);
}
// Kernel specialisations.  A kernel that inlines every (op, rows per unit)
// matvec variant compiles its hot loop worse (measured: 1.2 vs 0.65 us per page);
// shapes whose units all have the same row count and whose attention has one
// known form get a kernel with only those variants inlined.
//   SPEC 0  any shape: variants dispatched at run time, out of line
//   SPEC 1  4-row units, head_dim 64, 4 query heads per kv head, bf16 KV (Llama-3.2-1B)
//   SPEC 2  2-row units, head_dim 128, 4 query heads per kv head, fp16 KV (Llama-3-8B)
template <int SPEC> struct Spec;
template <> struct Spec<1> { static constexpr int rt = 4, dh = 64, rep = 4; static constexpr bool kv16 = false; };
template <> struct Spec<2> { static constexpr int rt = 2, dh = 128, rep = 4; static constexpr bool kv16 = true; };

template <int OPK, int NBT, int SPEC>
__device__ __forceinline__ void mv_dispatch(int rt, const KParams& p, const Instr& I, uint32_t pb,
                                            uint8_t* ring, const float* act, int K, uint64_t* full,
                                            uint64_t* empty, Misc* misc, uint32_t ii) {
  if constexpr (SPEC != 0) {
    mv_run<OPK, Spec<SPEC>::rt, NBT>(p, I, pb, ring, act, K, full, empty, misc, ii);
  } else {
    switch (rt) {
      case 1: if constexpr (OPK == OP_O || OPK == OP_DOWN || OPK == OP_LM) mv_units_call<OPK, 1, NBT>(p, I, pb, ring, act, K, full, empty, misc, ii); break;
      case 2: mv_units_call<OPK, 2, NBT>(p, I, pb, ring, act, K, full, empty, misc, ii); break;
      case 4: mv_units_call<OPK, 4, NBT>(p, I, pb, ring, act, K, full, empty, misc, ii); break;
      case 8: mv_units_call<OPK, 8, NBT>(p, I, pb, ring, act, K, full, empty, misc, ii); break;
    }
  }
}

template <int DH, bool KV16F>
__device__ __forceinline__ uint32_t attn_dispatch_rep(const KParams& p, const Instr& I, uint32_t pb,
                                                      uint8_t* ring, float* act, uint64_t* full,
                                                      uint64_t* empty, Misc* misc, uint32_t ii) {
  switch (p.D.rep) {
    case 1: return attn_units<DH, 1, KV16F>(p, I, pb, ring, act, full, empty, misc, ii);
    case 2: return attn_units<DH, 2, KV16F>(p, I, pb, ring, act, full, empty, misc, ii);
    case 4: return attn_units<DH, 4, KV16F>(p, I, pb, ring, act, full, empty, misc, ii);
    default: return attn_units<DH, 8, KV16F>(p, I, pb, ring, act, full, empty, misc, ii);
  }
}
template <int DH>
__device__ __forceinline__ uint32_t attn_dispatch(const KParams& p, const Instr& I, uint32_t pb,
                                                  uint8_t* ring, float* act, uint64_t* full,
                                                  uint64_t* empty, Misc* misc, uint32_t ii) {
  return p.D.kv_fp16 ? attn_dispatch_rep<DH, true>(p, I, pb, ring, act, full, empty, misc, ii)
                     : attn_dispatch_rep<DH, false>(p, I, pb, ring, act, full, empty, misc, ii);
}

template <int NBT, int SPEC>
static __device__ __noinline__ void consumer(const KParams& p, uint8_t* ring, float* act, uint64_t* full,
                                      uint64_t* empty, Misc* misc) {
  const Dims& D = p.D;
  const int ct = threadIdx.x - 32;
  const uint32_t i0 = p.sm_off[blockIdx.x], i1 = p.sm_off[blockIdx.x + 1];
  uint32_t page_base = 0;
  const int half = D.d / 2;
  // tensor-core units: the 8-lane kernel of the Llama-3.2-1B shape family holds two
  // accumulator buffers (kTcCols fp32 columns) in tensor memory for the whole launch
  constexpr bool kTC = NBT == 8 && SPEC == 1;
  uint32_t tc_n = 0;
  if constexpr (kTC) {
    if (ct < 32) tmem_alloc(&misc->tmem_base, kTcCols);
    tc_fence_before();
    cbar();
    tc_fence_after();
  }
  for (int t = 0; t < p.n_steps; ++t) {
  // step t begins once step t - 1 has written its ids everywhere (acquire): its
  // tokens, every read of its activations and every write of its KV rows are done
  if (ct == 0) {
    misc->step = t;
    misc->i0 = i0;
    misc->n_instr = i1 - i0;
    misc->actset = p.acts + (size_t)((p.parity0 + t) & 1) * p.set_floats;
    if (t > 0 && !wait_counter(p, p.ctr + ctr_step(D), (uint32_t)t, i0)) misc->stop = 1;
    // a (lane, kv head) split by query head signals once per head (attn_plan)
    uint32_t extra = 0;
    for (int b = 0; b < p.nb; ++b)
      if (attn_plan(p.S, D.rep, (p.pos[b] + t) / D.PL + 1, 0).single) extra += (uint32_t)(D.Hkv * (D.rep - 1));
    misc->attn_extra += extra;
  }
  cbar();
  if (misc->stop) break;
  // per-step constants: positions, tokens, RoPE (cos, sin) at each lane's
  // position, and the KV page that position lives in
  if (ct < p.nb) {
    misc->pos[ct] = p.pos[ct] + t;
    misc->cur_phys[ct] = p.page_table[p.slot[ct] * D.pages_per_seq + (p.pos[ct] + t) / D.PL];
  }
  if (ct < NBT) {
    const int* step_tokens = (p.chain && t > 0) ? p.ids + (size_t)(t - 1) * p.ids_stride
                                                : p.tokens + (size_t)(p.chain ? 0 : t) * p.nb;
    int tk = ct < p.nb ? __ldcg(step_tokens + ct) : 0;  // may be written in this launch
    if (tk < 0 || tk >= D.V) {
      raise_error(p, E_BAD_TOKEN, i0, (uint32_t)tk, false);
      tk = 0;
    }
    misc->tok[ct] = tk;
  }
  for (int e = ct; e < p.nb * half; e += 256) {
    const int b = e / half, i = e % half;
    misc->rope_cs[b][i] = p.rope[(size_t)(p.pos[b] + t) * half + i];
  }
  {  // refill this SM's share of the other activation set: sentinel, accumulators zero
    uint4* other = reinterpret_cast<uint4*>(p.acts + (size_t)((p.parity0 + t + 1) & 1) * p.set_floats);
    const long long n4 = p.set_floats / 4, per = (n4 + gridDim.x - 1) / gridDim.x, acc4 = p.acc_base / 4;
    const long long lo = (long long)blockIdx.x * per, hi = min(n4, lo + per);
    const uint4 sv = make_uint4(kSentinel, kSentinel, kSentinel, kSentinel), zv = make_uint4(0u, 0u, 0u, 0u);
    for (long long e = lo + ct; e < hi; e += 256) st_relaxed_u4(other + e, e < acc4 ? sv : zv);
  }
  cbar();
  bool stopped = false;  // set only where every warp reads misc->stop together
  long long* prev_rec = nullptr;  // profile: record whose re-read counters await their flush
  Instr I;
  if (i0 < i1) I = p.instrs[i0];
  for (uint32_t ii = i0; ii < i1; ++ii) {
    const Instr In = ii + 1 < i1 ? p.instrs[ii + 1] : I;  // loaded while this one runs
    long long* rec = (p.prof && ct == 0) ? p.prof + ((size_t)blockIdx.x * p.prof_stride + (ii - i0)) * kProfSlots : nullptr;
    // The next instruction's RMSNorm gain is read once per step: pull it into L2
    // now, so its staging does not start behind a DRAM miss.
    if ((In.op == OP_QKV || In.op == OP_GU || In.op == OP_LM) && ct < 32 && ct * 64 < D.H)
      prefetch_l2(static_cast<const uint16_t*>(In.ptr[3]) + ct * 64);
    if (rec) {
      rec[0] = (long long)I.op | ((long long)I.layer << 8) | ((long long)I.n_units << 24);
      rec[1] = (long long)globaltimer_ns();
    }
    if (ct == 0 && I.dep != kNoCounter && ((p.hints >> I.op) & 1)) {
      // hint: every warp of a matvec instruction bumps its counter, attention once
      // per (lane, kv head); counters only grow within a launch
      const uint32_t per = I.op == OP_O ? 1u : (uint32_t)kConsumerWarps;
      const uint32_t extra = I.op == OP_O ? misc->attn_extra : 0u;
      if (!wait_hint(p, p.ctr + I.dep, I.dep_target * per * (uint32_t)(t + 1) + extra, ii)) misc->stop = 1;
    }
    cbar();
    if (ct == 0) misc->cons_seq = (uint32_t)t * misc->n_instr + (ii - i0);  // entered (dynamic-tail table)
    if (rec) rec[2] = (long long)globaltimer_ns();
    if (prev_rec) {  // every warp is past the previous instruction now (reductions: no wait)
      atomicAdd(reinterpret_cast<unsigned long long*>(prev_rec + 16), (unsigned long long)misc->slow_n);
      atomicAdd(reinterpret_cast<unsigned long long*>(prev_rec + 17), misc->slow_ns);
      misc->slow_n = 0;
      misc->slow_ns = 0;
      prev_rec = nullptr;
    }
    if (misc->stop) { stopped = true; break; }
    float* lay = misc->actset + (size_t)I.layer * p.layer_floats;
    uint32_t used = I.n_units;  // one page per unit, except attention
    switch (I.op) {
      case OP_QKV: {
        const uint16_t* gain = static_cast<const uint16_t*>(I.ptr[3]);
        if (I.layer == 0)
          stage<NBT, ST_EMB, true>(p, act, misc, nullptr, 0, D.H, gain, ii);
        else
          stage<NBT, ST_ACC, true>(p, act, misc, reinterpret_cast<const float*>(acc_of(p, misc, I.layer - 1)),
                                   D.H, D.H, gain, ii);
        if (rec) rec[11] = (long long)globaltimer_ns();
        mv_dispatch<OP_QKV, NBT, SPEC>(2 * D.RP, p, I, page_base, ring, act, D.H, full, empty, misc, ii);
        break;
      }
      case OP_ATTN:
        if constexpr (SPEC != 0 && NBT <= 2)  // inlined in the specialised kernels (no call spills)
          used = attn_units_body<Spec<SPEC>::dh, Spec<SPEC>::rep, Spec<SPEC>::kv16>(p, I, page_base, ring, act,
                                                                                    full, empty, misc, ii);
        else if constexpr (SPEC != 0)
          used = attn_units<Spec<SPEC>::dh, Spec<SPEC>::rep, Spec<SPEC>::kv16>(p, I, page_base, ring, act, full,
                                                                               empty, misc, ii);
        else
          used = D.d == 64 ? attn_dispatch<64>(p, I, page_base, ring, act, full, empty, misc, ii)
                           : attn_dispatch<128>(p, I, page_base, ring, act, full, empty, misc, ii);
        break;
      case OP_O:
        stage<NBT, ST_ONE, false>(p, act, misc, lay + p.off_o, D.qdim, D.qdim, nullptr, ii);
        if (rec) rec[11] = (long long)globaltimer_ns();
        mv_dispatch<OP_O, NBT, SPEC>(D.Ro, p, I, page_base, ring, act, D.qdim, full, empty, misc, ii);
        break;
      case OP_GU:
        stage<NBT, ST_ONE, true>(p, act, misc, lay + p.off_x1, D.H, D.H, static_cast<const uint16_t*>(I.ptr[3]), ii);
        if (rec) rec[11] = (long long)globaltimer_ns();
        mv_dispatch<OP_GU, NBT, SPEC>(2 * D.Rgu, p, I, page_base, ring, act, D.H, full, empty, misc, ii);
        break;
      case OP_DOWN:
        stage<NBT, ST_ONE, false>(p, act, misc, lay + p.off_a + (size_t)I.arg * D.KS, D.F, D.KS, nullptr, ii);
        if (rec) rec[11] = (long long)globaltimer_ns();
        mv_dispatch<OP_DOWN, NBT, SPEC>(D.Rdn, p, I, page_base, ring, act, D.KS, full, empty, misc, ii);
        break;
      case OP_LM:
        stage<NBT, ST_ACC, true>(p, act, misc, reinterpret_cast<const float*>(acc_of(p, misc, D.L - 1)), D.H,
                                 D.H, static_cast<const uint16_t*>(I.ptr[3]), ii);
        if (rec) rec[11] = (long long)globaltimer_ns();
        mv_dispatch<OP_LM, NBT, SPEC>(D.Rlm, p, I, page_base, ring, act, D.H, full, empty, misc, ii);
        break;
      case OP_GU_TC:
        if constexpr (kTC) {
          stage<NBT, ST_ONE, true, true>(p, act, misc, lay + p.off_x1, D.H, D.H,
                                         static_cast<const uint16_t*>(I.ptr[3]), ii);
          if (rec) rec[11] = (long long)globaltimer_ns();
          mv_units_tc<OP_GU_TC>(p, I, page_base, ring, act, full, empty, misc, ii, tc_n);
          used = I.n_units * (uint32_t)D.nkt;
        }
        break;
      case OP_LM_TC:
        if constexpr (kTC) {
          stage<NBT, ST_ACC, true, true>(p, act, misc, reinterpret_cast<const float*>(acc_of(p, misc, D.L - 1)),
                                         D.H, D.H, static_cast<const uint16_t*>(I.ptr[3]), ii);
          if (rec) rec[11] = (long long)globaltimer_ns();
          mv_units_tc<OP_LM_TC>(p, I, page_base, ring, act, full, empty, misc, ii, tc_n);
          used = I.n_units * (uint32_t)D.nkt;
        }
        break;
    }
    if (I.pool) used = (uint32_t)misc->dyn_end[((uint32_t)t * misc->n_instr + (ii - i0)) & 15] - page_base;
    page_base += used;
    // No barrier here: each warp bumped the hint counter after its own writes,
    // and the next instruction's barrier keeps the activation buffer from being
    // restaged while a warp still reads it.  Profiling stamps without a barrier
    // too: every warp raises the record's end times to its own.
    if (p.prof) {
      const long long now = (long long)globaltimer_ns();
      long long* rw = p.prof + ((size_t)blockIdx.x * p.prof_stride + (ii - i0)) * kProfSlots;
      if ((ct & 31) == 0) {
        unsigned long long* ru = reinterpret_cast<unsigned long long*>(rw);
        if (I.op != OP_ATTN) atomicMax(ru + 12, (unsigned long long)now);
        atomicMax(ru + 13, (unsigned long long)now);
        atomicMax(ru + 4, (unsigned long long)now);
      }
      if (rec) {
        rec[3] = now;
        if (I.op != OP_ATTN) { rec[18] = misc->t_stage_in; rec[19] = misc->t_stage_loaded; }
        if (I.op == OP_LM || (I.op == OP_QKV && I.layer > 0)) { rec[20] = misc->t_sum_x1; rec[21] = misc->t_sum_p; }
        if (I.op != OP_ATTN) { rec[22] = misc->warp_entry[0]; rec[24] = misc->warp_first[0]; }
        prev_rec = rec;  // its re-read counters are flushed once every warp is past it
      }
    }
    I = In;
  }
  if (stopped) break;
  // a stop raised later in this step is acted on after the next step's barrier,
  // where every warp reads the flag at the same point
  }
  if constexpr (kTC) {  // every MMA has completed (its accumulator was read back)
    tc_fence_before();
    cbar();
    tc_fence_after();
    if (ct < 32) tmem_dealloc(misc->tmem_base, kTcCols);
  }
}

// ---------------------------------------------------------------- the kernel

template <int NBT, int SPEC>
__global__ void __launch_bounds__(kThreads, 1) mk_decode_kernel(const __grid_constant__ KParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Misc* misc = reinterpret_cast<Misc*>(smem + p.misc_off);
  static_assert(sizeof(KParams) % 4 == 0, "KParams copy");
  for (int i = threadIdx.x; i < (int)(sizeof(KParams) / 4); i += kThreads)
    reinterpret_cast<uint32_t*>(&misc->kp)[i] = reinterpret_cast<const uint32_t*>(&p)[i];
  // Ring protocol.  Page i (in this SM's stream order) goes to slot i % NP and
  // completes full barrier i % (2 NP), phase parity (i / (2 NP)) & 1; its slot is
  // released on empty barrier i % NP by 8 warp arrivals.  A consumer only waits on
  // page i after page i - NP was issued (NP >= 8 consumer warps, each taking
  // pages in order), so page i - 2 NP -- the previous user of the same full
  // barrier -- has been consumed and the parity wait cannot alias an older phase,
  // even when bulk copies land out of order.
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
  uint64_t* empty = full + 128;
  // the next step's counters start from zero (this step's were zeroed by the previous one)
  for (int i = blockIdx.x * kThreads + threadIdx.x; i < p.n_counters; i += gridDim.x * kThreads)
    p.ctr_next[i] = 0u;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * p.ring_pages; ++i) mbar_init(&full[i], 1);
    for (int i = 0; i < p.ring_pages; ++i) mbar_init(&empty[i], kConsumerWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&misc->tc_accf[i], 1);
      mbar_init(&misc->tc_acce[i], 4);  // the four epilogue warps
    }
    fence_barrier_init();
    fence_proxy_async_smem();
    misc->stop = 0;
    misc->last = 0;
    misc->issued = 0;
    misc->entry_abort = aborted(p) ? 1 : 0;
    misc->slow_n = 0;
    misc->slow_ns = 0;
    misc->attn_extra = 0;
    misc->cons_seq = 0;
    for (int i = 0; i < 16; ++i) misc->dyn_end[i] = ~0ull;  // a tag no instruction has
  }
  __syncthreads();
  if (!misc->entry_abort) {
    const int warp = threadIdx.x >> 5;
    if (warp == 0) {
      if (threadIdx.x == 0) producer(misc->kp, smem, full, empty, misc);
    } else if (warp <= kConsumerWarps) {
      consumer<NBT, SPEC>(misc->kp, smem, reinterpret_cast<float*>(smem + p.act_off), full, empty, misc);
    }
  }
  __syncthreads();
}

}  // namespace mk
