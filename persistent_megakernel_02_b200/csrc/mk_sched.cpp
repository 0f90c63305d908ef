// mk_sched.cpp -- host scheduler: lowers a decoder shape into per-SM instruction
// tapes with counter targets, and a CPU simulator that runs a tape to prove it is
// deadlock-free, covers every output exactly once and waits on full fan-in.
//
// The Hazy megakernel article (section "Megakernel: a deep-fusion design from
// scratch") says the dependencies between instructions are analysed and laid
// out before the run, and each SM gets its own ordered execution plan; the
// forum post "Two thousand four hundred kernel launches per token" (tail-effect
// example: 512 work blocks on 148 SMs leave 80 idle in the last wave) is why
// units are assigned by cumulative bytes per SM rather than in waves.
#include <algorithm>
#include <cstdio>
#include <queue>
#include <string>
#include <vector>

#include "mk_plan.h"

namespace mk {

static int pow2_floor(long long x) {
  if (x < 1) return 1;
  int p = 1;
  while ((long long)p * 2 <= x) p *= 2;
  return p;
}

// rows of length k (bf16) that fit one page, at most 8, a power of two
static int page_rows(int k) { return std::min(8, pow2_floor(kPageBytes / (2LL * k))); }

std::string derive_dims(int n_layers, int hidden, int n_heads, int n_kv_heads, int head_dim,
                        int ffn, int vocab, int tied, float eps, int max_batch, int max_seq,
                        int n_sm, Dims* out) {
  char buf[256];
  if (n_layers < 1 || n_layers > 4096) return "n_layers out of range";
  if (head_dim != 64 && head_dim != 128) return "head_dim must be 64 or 128";
  if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads) return "n_heads must be a multiple of n_kv_heads";
  int rep = n_heads / n_kv_heads;
  if (rep != 1 && rep != 2 && rep != 4 && rep != 8) return "n_heads / n_kv_heads must be 1, 2, 4 or 8";
  if (n_kv_heads > 255) return "n_kv_heads too large";
  if (hidden < 8 || hidden % 8) return "hidden must be a positive multiple of 8";
  if (hidden > 4096) return "hidden > 4096 is not supported (two rows per 16 KiB page)";
  if (ffn < 8 || ffn % 8) return "ffn must be a positive multiple of 8";
  int qdim = n_heads * head_dim, kvdim = n_kv_heads * head_dim;
  if (qdim > 8192) return "n_heads * head_dim > 8192 is not supported";
  if (vocab < 1) return "vocab must be positive";
  if (max_batch < 1 || max_batch > kMaxNB) return "max_batch must be in 1..8";
  if (max_seq < 1 || max_seq > (1 << 24)) return "max_seq out of range";
  if (n_sm < 1 || n_sm > 4096) return "n_sm out of range";
  int kact = std::max(hidden, qdim);
  int nbt = lanes_template(max_batch);
  if ((long long)nbt * kact > kActFloatsMax) {
    snprintf(buf, sizeof buf,
             "max_batch (rounded up to %d) * max(hidden, n_heads*head_dim) = %lld exceeds %d", nbt,
             (long long)nbt * kact, kActFloatsMax);
    return buf;
  }
  Dims D{};
  D.L = n_layers; D.H = hidden; D.Hq = n_heads; D.Hkv = n_kv_heads; D.d = head_dim;
  D.F = ffn; D.V = vocab; D.qdim = qdim; D.kvdim = kvdim; D.rep = rep;
  D.eps = eps; D.tied = tied ? 1 : 0;
  D.max_batch = max_batch; D.max_seq = max_seq;
  // down projection: K slices no wider than the staged activation
  int n_ks = 0;
  for (int n = std::max(1, (ffn + kact - 1) / kact); n <= ffn / 8; ++n) {
    if (ffn % n == 0 && (ffn / n) % 8 == 0 && ffn / n <= kact) { n_ks = n; break; }
  }
  if (!n_ks) return "ffn cannot be split into K slices of at most max(hidden, qdim)";
  D.n_ks = n_ks; D.KS = ffn / n_ks;
  if (n_ks > kMaxKS) return "ffn needs more than 8 down-projection K slices";
  // rows per unit: as many as fit a page, but no more than keep every SM busy
  long long pairs = (long long)(n_heads + 2 * n_kv_heads) * (head_dim / 2);
  D.RP = std::min(page_rows(hidden) / 2, pow2_floor(pairs / n_sm));
  if (D.RP < 1) D.RP = 1;
  while ((head_dim / 2) % D.RP) D.RP /= 2;
  D.Ro = std::min(page_rows(qdim), pow2_floor(hidden / n_sm));
  D.Rgu = std::max(1, std::min(page_rows(hidden) / 2, pow2_floor(ffn / n_sm)));
  D.Rdn = std::min(page_rows(D.KS), pow2_floor((long long)hidden * n_ks / n_sm));
  D.Rlm = std::min(page_rows(hidden), pow2_floor(vocab / n_sm));
  D.PL = kPageBytes / (4 * head_dim);
  D.pages_per_seq = (max_seq + D.PL - 1) / D.PL;
  D.n_phys_pages = max_batch * D.pages_per_seq;
  D.n_qkv = (int)(pairs / D.RP);
  D.n_o = (hidden + D.Ro - 1) / D.Ro;
  D.n_gu = (ffn + D.Rgu - 1) / D.Rgu;
  D.n_dn = (hidden + D.Rdn - 1) / D.Rdn;
  D.n_lm = (vocab + D.Rlm - 1) / D.Rlm;
  D.tc = 0;  // enabled by the handle when its kernels can run the tensor-core units
  D.nkt = hidden / 64;
  D.n_gu_tc = ffn / 64;
  D.n_lm_tc = (vocab + 127) / 128;
  if (n_counters(D) >= kNoCounter) return "too many counters for this shape";
  *out = D;
  return "";
}

// Attention units per (lane, kv head): as many as the SMs allow, but no more than
// there is work for -- a slice per KV page for long contexts, and for short ones
// (the kernel's head split, attn_plan) one unit per query head, so at least rep
// even where a sequence has fewer pages than its kv head has query heads (short
// max_seq); capping that at the page count disabled the head split (Llama-3.2-1B
// batch 1 with max_seq 93: 487 us/step instead of 456).
int attn_slices(const Dims& D, int n_sm, int nb) {
  int s = n_sm / (nb * D.Hkv);
  s = std::max(1, std::min(s, std::max(D.pages_per_seq, D.rep)));
  return std::min(s, 65535);
}

// bytes one unit streams (weights), or an estimate for an attention slice
static int64_t unit_bytes(const Dims& D, int op, int S) {
  switch (op) {
    case OP_QKV: return 2LL * 2 * D.RP * D.H;
    case OP_O: return 2LL * D.Ro * D.qdim;
    case OP_GU: return 2LL * 2 * D.Rgu * D.H;
    case OP_DOWN: return 2LL * D.Rdn * D.KS;
    case OP_LM: return 2LL * D.Rlm * D.H;
    case OP_GU_TC:
    case OP_LM_TC: return (int64_t)D.nkt * kPageBytes;
    case OP_ATTN: {
      int pages = (D.pages_per_seq + S - 1) / S;
      return (int64_t)pages * kPageBytes;
    }
  }
  return 0;
}

namespace {
struct Assigner {
  std::vector<int64_t>& load;
  explicit Assigner(std::vector<int64_t>& l) : load(l) {}
  // Split n equal units over the SMs of [lo, hi): how many each SM gets is decided
  // by cumulative bytes (the least-loaded SM takes the next unit, ties: lowest
  // id), and each SM receives a CONTIGUOUS range of units, in SM order.  Keeping
  // an SM's weights of one phase contiguous keeps its bulk copies within a few
  // GPU pages instead of one new page per copy.
  std::vector<std::vector<uint32_t>> run(int n, int64_t bytes, int lo, int hi) {
    using E = std::pair<int64_t, int>;
    std::priority_queue<E, std::vector<E>, std::greater<E>> pq;
    for (int s = lo; s < hi; ++s) pq.push({load[s], s});
    std::vector<int> count(load.size(), 0);
    for (int u = 0; u < n; ++u) {
      E e = pq.top();
      pq.pop();
      count[e.second]++;
      e.first += bytes;
      load[e.second] = e.first;
      pq.push(e);
    }
    std::vector<std::vector<uint32_t>> out(load.size());
    uint32_t u = 0;
    for (int s = lo; s < hi; ++s)
      for (int c = 0; c < count[s]; ++c) out[s].push_back(u++);
    return out;
  }
};
}  // namespace

Tape lower(const Dims& D, int n_sm, int nb, int dyn_percent, int region) {
  Tape t;
  t.nb = nb;
  t.region = region;
  // 5-8 lanes run the 8-lane kernel, whose LM head (bit 0) and gate/up (bit 1) may
  // use the tensor cores
  t.tc = lanes_template(nb) == 8 ? D.tc : 0;
  t.S = attn_slices(D, n_sm, nb);
  t.n_counters = n_counters(D);
  std::vector<int64_t> load(n_sm, 0);
  Assigner as(load);
  std::vector<std::vector<Instr>> ins(n_sm);

  // units must form one contiguous range per instruction (the Assigner's output)
  auto emit = [&](int sm, uint8_t op, int layer, const std::vector<uint32_t>& units, uint16_t dep,
                  uint16_t sig, uint8_t arg) -> Instr& {
    Instr I{};
    I.op = op; I.arg = arg; I.layer = (uint16_t)layer;
    I.u0 = units.empty() ? 0u : units[0];
    I.n_units = (uint32_t)units.size();
    for (size_t k = 1; k < units.size(); ++k)
      if (units[k] != units[0] + k) I.n_units = 0xFFFFFFFFu;  // not a range: simulate() reports it
    I.dep = dep; I.sig = sig; I.dep_target = 0;
    ins[sm].push_back(I);
    return ins[sm].back();
  };

  // A streaming phase over SMs [lo, hi): the first units are split statically
  // (contiguous ranges), the last dyn_percent % form the pool the SMs claim from
  // in chunks.  Every SM of the range gets an instruction when there is a pool.
  dyn_percent = std::max(0, std::min(90, dyn_percent));
  auto phase = [&](uint8_t op, int layer, int n, int lo, int hi, uint16_t dep, uint16_t sig, uint8_t arg,
                   int pool, bool every_sm) {
    const int n_part = hi - lo;
    const int n_dyn = pool >= 0 ? (int)((int64_t)n * dyn_percent / 100) : 0;
    const int n_st = n - n_dyn;
    const int64_t ub = unit_bytes(D, op, t.S);
    // Gate/up tensor-core blocks are 32 pages each and fewer than the SMs: counted
    // in the cumulative load they would hand the SMs without one extra units of
    // every later phase, and those SMs would lead the latency-bound phases.  They
    // take the least-loaded SMs without changing the balance of the rest.
    const std::vector<int64_t> saved = op == OP_GU_TC ? load : std::vector<int64_t>();
    auto st = as.run(n_st, ub, lo, hi);
    if (op == OP_GU_TC) load = saved;
    // each SM's expected share of the pool counts toward its load
    if (n_dyn > 0)
      for (int s = lo; s < hi; ++s) load[s] += ub * n_dyn / n_part;
    // chunks small enough that the last ones balance the SMs' end times, at least
    // two units where the pool has them (a claim is a round trip to L2)
    const int per_sm = n_dyn / std::max(1, n_part);
    const uint32_t chunk = (uint32_t)std::max(per_sm >= 4 ? 2 : 1, std::min(4, per_sm / 8));
    for (int s = lo; s < hi; ++s)
      if (!st[s].empty() || n_dyn > 0 || every_sm) {
        Instr& I = emit(s, op, layer, st[s], dep, sig, arg);
        if (n_dyn > 0) {
          I.pool = (uint32_t)(pool + 1) | (chunk << 24);
          I.pool_u0 = (uint32_t)n_st;
          I.pool_u1 = (uint32_t)n;
        }
      }
  };

  for (int l = 0; l < (region == REGION_LM ? 0 : D.L); ++l) {
    uint16_t dep_qkv = l ? (uint16_t)ctr_layer(l - 1, C_DOWN) : kNoCounter;
    // RMSNorm + QKV + RoPE
    auto a = as.run(D.n_qkv, unit_bytes(D, OP_QKV, t.S), 0, n_sm);
    for (int s = 0; s < n_sm; ++s)
      if (!a[s].empty()) emit(s, OP_QKV, l, a[s], dep_qkv, (uint16_t)ctr_layer(l, C_QKV), 0);
    // attention slices (lane, kv head, slice)
    {
      int n = nb * D.Hkv * t.S;
      auto at = as.run(n, unit_bytes(D, OP_ATTN, t.S), 0, n_sm);
      for (int s = 0; s < n_sm; ++s)
        if (!at[s].empty()) emit(s, OP_ATTN, l, at[s], (uint16_t)ctr_layer(l, C_QKV), kNoCounter, 0);
    }
    // O projection + residual
    auto o = as.run(D.n_o, unit_bytes(D, OP_O, t.S), 0, n_sm);
    for (int s = 0; s < n_sm; ++s)
      if (!o[s].empty()) emit(s, OP_O, l, o[s], (uint16_t)ctr_layer(l, C_ATTN), (uint16_t)ctr_layer(l, C_O), 0);
    // RMSNorm + gate/up + SwiGLU
    if (t.tc & 2)
      phase(OP_GU_TC, l, D.n_gu_tc, 0, n_sm, (uint16_t)ctr_layer(l, C_O), (uint16_t)ctr_layer(l, C_GU), 0, -1,
            false);
    else
      phase(OP_GU, l, D.n_gu, 0, n_sm, (uint16_t)ctr_layer(l, C_O), (uint16_t)ctr_layer(l, C_GU), 0,
            pool_gu(D, l), false);
    // down projection + residual: SMs split into one group per K slice
    for (int ks = 0; ks < D.n_ks; ++ks) {
      int lo = (int)((long long)n_sm * ks / D.n_ks), hi = (int)((long long)n_sm * (ks + 1) / D.n_ks);
      if (hi <= lo) hi = lo + 1;  // more slices than SMs: share
      lo %= n_sm; hi = std::min(hi, n_sm);
      phase(OP_DOWN, l, D.n_dn, lo, hi, (uint16_t)ctr_layer(l, C_GU), (uint16_t)ctr_layer(l, C_DOWN),
            (uint8_t)ks, pool_dn(D, l, ks), false);
    }
  }
  // final norm + LM head + argmax: every SM takes part (possibly with no rows)
  // (in its own launch it waits on nothing: the launch boundary orders it)
  if (region != REGION_LAYERS)
    phase((t.tc & 1) ? OP_LM_TC : OP_LM, D.L, (t.tc & 1) ? D.n_lm_tc : D.n_lm, 0, n_sm,
          region == REGION_LM ? kNoCounter : (uint16_t)ctr_layer(D.L - 1, C_DOWN), kNoCounter, 0,
          (t.tc & 1) ? -1 : pool_lm(D), true);

  // wait targets = how many instructions signal the counter in one step
  std::vector<uint32_t> fan(t.n_counters, 0);
  for (int s = 0; s < n_sm; ++s)
    for (auto& I : ins[s])
      if (I.sig != kNoCounter) fan[I.sig]++;
  for (int l = 0; l < D.L; ++l) fan[ctr_layer(l, C_ATTN)] = (uint32_t)(nb * D.Hkv);
  for (int s = 0; s < n_sm; ++s)
    for (auto& I : ins[s])
      if (I.dep != kNoCounter) I.dep_target = fan[I.dep];

  // concatenate
  t.sm_off.assign(n_sm + 1, 0);
  for (int s = 0; s < n_sm; ++s) {
    t.sm_off[s] = (uint32_t)t.instrs.size();
    t.instrs.insert(t.instrs.end(), ins[s].begin(), ins[s].end());
  }
  t.sm_off[n_sm] = (uint32_t)t.instrs.size();
  return t;
}

SimReport simulate(const Dims& D, int n_sm, const Tape& t) {
  SimReport r;
  std::vector<int64_t> ctr(t.n_counters, 0), signals(t.n_counters, 0);
  std::vector<int64_t> part((size_t)D.L * kMaxNB * D.Hkv, 0);
  const int nb = t.nb, S = t.S;
  // coverage: per layer and op, how often each output tile was produced
  std::vector<int> cq((size_t)D.L * D.n_qkv, 0), co((size_t)D.L * D.n_o, 0),
      cg((size_t)D.L * D.n_gu, 0), cd((size_t)D.L * D.n_ks * D.n_dn, 0),
      ca((size_t)D.L * nb * D.Hkv * S, 0), cl(D.n_lm, 0);
  // tensor-core tapes cover gate/up and/or the LM head in 128-row blocks instead
  if (t.tc & 2) cg.assign((size_t)D.L * D.n_gu_tc, 0);
  if (t.tc & 1) cl.assign(D.n_lm_tc, 0);
  std::vector<uint32_t> ip(n_sm);
  r.bytes_min = INT64_MAX; r.bytes_max = 0;
  // SMs taking part in each pool: each is expected to stream an equal share of it
  std::vector<int64_t> pool_part(n_pools(D), 0);
  for (const Instr& I : t.instrs)
    if (I.pool && (I.pool & 0xFFFFFFu) - 1 < pool_part.size()) pool_part[(I.pool & 0xFFFFFFu) - 1]++;
  for (int s = 0; s < n_sm; ++s) {
    ip[s] = t.sm_off[s];
    int n = (int)(t.sm_off[s + 1] - t.sm_off[s]);
    r.max_instr_per_sm = std::max(r.max_instr_per_sm, n);
    int64_t by = 0;
    for (uint32_t i = t.sm_off[s]; i < t.sm_off[s + 1]; ++i) {
      const Instr& I = t.instrs[i];
      if (I.n_units != 0xFFFFFFFFu) by += unit_bytes(D, I.op, S) * I.n_units;
      if (I.pool && (I.pool & 0xFFFFFFu) - 1 < pool_part.size() && I.pool_u1 >= I.pool_u0)
        by += unit_bytes(D, I.op, S) * (I.pool_u1 - I.pool_u0) / pool_part[(I.pool & 0xFFFFFFu) - 1];
    }
    r.bytes_min = std::min(r.bytes_min, by);
    r.bytes_max = std::max(r.bytes_max, by);
  }
  r.n_instr_total = (int)t.instrs.size();
  bool cover_err = false;
  auto bump = [&](std::vector<int>& v, size_t i) {
    if (i >= v.size()) { cover_err = true; return; }
    v[i]++;
  };
  // a pool's units are produced once, by whichever SMs claim them: the simulator
  // credits them when the first instruction of the pool runs
  std::vector<char> pool_seen(n_pools(D), 0);
  std::vector<int64_t> pool_range(n_pools(D), -1);
  bool progress = true;
  while (progress) {
    progress = false;
    for (int s = 0; s < n_sm; ++s) {
      while (ip[s] < t.sm_off[s + 1]) {
        const Instr& I = t.instrs[ip[s]];
        if (I.dep != kNoCounter && ctr[I.dep] < (int64_t)I.dep_target) break;
        int l = I.layer;
        if (I.n_units == 0xFFFFFFFFu) { cover_err = true; ip[s]++; progress = true; continue; }
        uint32_t n_run = I.n_units;
        std::vector<uint32_t> extra;
        if (I.pool) {
          const uint32_t pi = (I.pool & 0xFFFFFFu) - 1, chunk = I.pool >> 24;
          const int64_t key = ((int64_t)I.pool_u0 << 32) | I.pool_u1;
          const bool op_ok = I.op == OP_GU || I.op == OP_DOWN || I.op == OP_LM;
          if (!op_ok || pi >= pool_seen.size() || chunk < 1 || I.pool_u0 > I.pool_u1 ||
              I.u0 + I.n_units > I.pool_u0 || (pool_range[pi] >= 0 && pool_range[pi] != key)) {
            cover_err = true;
          } else {
            pool_range[pi] = key;
            if (!pool_seen[pi]) {
              pool_seen[pi] = 1;
              for (uint32_t u = I.pool_u0; u < I.pool_u1; ++u) extra.push_back(u);
            }
          }
        }
        for (uint32_t k = 0; k < n_run + extra.size(); ++k) {
          uint32_t u = k < n_run ? I.u0 + k : extra[k - n_run];
          switch (I.op) {
            case OP_QKV: bump(cq, (size_t)l * D.n_qkv + u); break;
            case OP_O: bump(co, (size_t)l * D.n_o + u); break;
            case OP_GU: bump(cg, (size_t)l * D.n_gu + u); if (t.tc & 2) cover_err = true; break;
            case OP_GU_TC: bump(cg, (size_t)l * D.n_gu_tc + u); if (!(t.tc & 2)) cover_err = true; break;
            case OP_LM_TC: bump(cl, u); if (!(t.tc & 1)) cover_err = true; break;
            case OP_DOWN: bump(cd, ((size_t)l * D.n_ks + I.arg) * D.n_dn + u); break;
            case OP_LM: bump(cl, u); if (t.tc & 1) cover_err = true; break;
            case OP_ATTN: {
              int b, g, sl;
              attn_unit(u, D.Hkv, S, &b, &g, &sl);
              if (b >= nb || g >= D.Hkv || sl >= S) { cover_err = true; break; }
              bump(ca, (((size_t)l * nb + b) * D.Hkv + g) * S + sl);
              size_t pi = ((size_t)l * kMaxNB + b) * D.Hkv + g;
              ctr[ctr_part(D, l, b, g)]++;
              if (++part[pi] == S) { ctr[ctr_layer(l, C_ATTN)]++; signals[ctr_layer(l, C_ATTN)]++; }
              break;
            }
          }
        }
        if (I.op == OP_LM || I.op == OP_LM_TC) { ctr[ctr_lm(D)]++; signals[ctr_lm(D)]++; }
        if (I.sig != kNoCounter) { ctr[I.sig]++; signals[I.sig]++; }
        ip[s]++;
        progress = true;
      }
    }
  }
  r.deadlock_free = true;
  for (int s = 0; s < n_sm; ++s)
    if (ip[s] != t.sm_off[s + 1]) {
      r.deadlock_free = false;
      char b[128];
      snprintf(b, sizeof b, "SM %d stuck at instruction %u", s, ip[s] - t.sm_off[s]);
      r.error = b;
      break;
    }
  auto all_one = [](const std::vector<int>& v) {
    for (int x : v)
      if (x != 1) return false;
    return true;
  };
  r.coverage_ok = !cover_err && all_one(cq) && all_one(co) && all_one(cg) && all_one(cd) &&
                  all_one(ca) && all_one(cl);
  if (t.region != REGION_ALL) {  // each part covers its own ops once and the other's not at all
    auto all_zero = [](const std::vector<int>& v) {
      for (int x : v)
        if (x != 0) return false;
      return true;
    };
    const bool layers_ok = all_one(cq) && all_one(co) && all_one(cg) && all_one(cd) && all_one(ca);
    const bool layers_none = all_zero(cq) && all_zero(co) && all_zero(cg) && all_zero(cd) && all_zero(ca);
    r.coverage_ok = !cover_err && (t.region == REGION_LAYERS ? layers_ok && all_zero(cl) : layers_none && all_one(cl));
  }
  r.targets_ok = true;
  for (const Instr& I : t.instrs)
    if (I.dep != kNoCounter && signals[I.dep] != (int64_t)I.dep_target) r.targets_ok = false;
  if (signals[ctr_lm(D)] != (t.region == REGION_LAYERS ? 0 : n_sm)) r.targets_ok = false;
  if (!r.coverage_ok && r.error.empty()) r.error = "coverage";
  if (!r.targets_ok && r.error.empty()) r.error = "targets";
  return r;
}

SmemLayout smem_layout(const Dims& D, int nb_max, int max_dyn_smem, int want_pages) {
  SmemLayout s{};
  int act = nb_max * std::max(std::max(D.H, D.qdim), D.KS) * 4;
  // attention scratch: q (rep x d) and the per-warp partials (rep x (d + 2))
  int attn = D.rep * D.d * 4 + kConsumerWarps * D.rep * (D.d + 2) * 4;
  // single-head short-context attention: q, 256 probabilities, 16 reductions, 512 partials
  attn = std::max(attn, (D.d + 256 + 16 + 512) * 4);
  s.act_bytes = (std::max(act, attn) + 1023) / 1024 * 1024;
  int misc = 8192;  // mbarriers (128 full + 64 empty), reduction scratch, step constants
  // Ring depth against L1: for a model streamed from HBM (weights larger than
  // L2) with a small activation region (10 KiB: one lane of a 2048-wide model, or
  // its attention scratch) the deepest ring that fits measured fastest
  // (Llama-3.2-1B batch 1: 13 pages 462 us, 11 pages 469; 8192-token context 738
  // vs 747).  Otherwise a ring fitted to the 196 KiB carveout, which leaves a
  // larger L1, measured faster (batch 4, 32 KiB: 974 vs 998 us; 8B batch 1,
  // 19 KiB: 3309 vs 3373; an L2-resident 256-wide model: 44 vs 62).
  const int64_t layer_w = 2LL * D.H * (D.qdim + 2 * D.kvdim) + 2LL * D.qdim * D.H + 6LL * D.H * D.F;
  const int64_t weights = layer_w * D.L + 2LL * D.V * D.H;
  const bool deep = s.act_bytes <= 12 * 1024 && weights > (128LL << 20);
  const int kCarveout196 = 196 * 1024 - 1024;  // minus the per-CTA reserved KiB
  int cap = deep ? max_dyn_smem : std::min(max_dyn_smem, kCarveout196);
  int np = std::min(64, (cap - s.act_bytes - misc) / kPageBytes);
  if (np < kConsumerWarps) np = std::min(64, (max_dyn_smem - s.act_bytes - misc) / kPageBytes);
  // the ring protocol needs at least one page per consumer warp
  if (want_pages > 0) np = std::min(std::min(64, (max_dyn_smem - s.act_bytes - misc) / kPageBytes),
                                    std::max(want_pages, kConsumerWarps));
  s.ring_pages = np;
  s.bar_off = np * kPageBytes + s.act_bytes;
  s.misc_off = s.bar_off + 8 * (128 + 64);  // 2 NP full + NP empty barriers, NP <= 64
  s.total = np * kPageBytes + s.act_bytes + misc;
  return s;
}

}  // namespace mk
