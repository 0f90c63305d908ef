// mk_prefill.cu -- batched prefill of a prompt on the tcgen05 tensor cores.
//
// Prefill is GEMM-shaped (a tile of prompt tokens times a tile of weight rows),
// where decode is a stream of matvecs; "One Megakernel is Not Enough: Predicting
// Where to Cut for Streaming Inference" (section "Why where to cut matters more
// than whether to fuse") notes that a language model runs the prompt once and
// then decodes per token, and the two phases have different shapes.  Per chunk of
// at most `chunk` prompt tokens and per layer:
//
//   pf_norm_split   n = RMSNorm(x) * g, written as bf16 high and low parts
//   pf_gemm<QKV>    [q; k; v] = W_{q,k,v} n on tcgen05; RoPE on q and k, K and V
//                   rounded into the paged cache, q kept in fp32
//   pf_attn         causal GQA attention of the chunk's queries over the cache
//                   (positions 0 .. own), online softmax, CUDA cores
//   pf_gemm<RESID>  x += W_o o
//   pf_norm_split   n = RMSNorm(x) * g_mlp
//   pf_gemm<SWIGLU> a = silu(W_g n) * (W_u n), written as bf16 high and low parts
//   pf_gemm<RESID>  x += W_d a
//
// GEMM: one CTA per 128-token x 128-feature output tile.  Warp 0 streams K slices
// of 64 through a 4-stage ring with 2D TMA loads (128-byte swizzle): the
// activation tile's high and low bf16 parts and the weight tile; warp 1 issues
// tcgen05.mma (M = 128, N = 128, K = 16) twice per K step -- high and low part
// against the same weights, so the product keeps about 16 significant bits of
// the fp32 activations -- into an fp32 accumulator in tensor memory; warps 2-5
// read it back with tcgen05.ld (one token row per thread) and run the epilogue.
// Every wait is bounded; on timeout the kernel records an error in the handle's
// error word, raises its abort flag and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "mk_prefill.h"
#include "mk_tc.cuh"

namespace mk {

namespace {

constexpr int kGM = 128;                      // tokens per tile (MMA M)
constexpr int kGN = 128;                      // output features per tile (MMA N)
constexpr int kGK = 64;                       // K per stage: one 128-byte swizzle row of bf16
constexpr int kGStages = 4;
constexpr int kGTile = kGM * kGK * 2;         // 16 KiB
constexpr int kGStageBytes = 3 * kGTile;      // activation high part, low part, weights
constexpr int kGThreads = 192;                // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kGSmem = 1024 + kGStages * kGStageBytes + 256;
constexpr uint32_t kGIdesc = idesc_bf16(kGM, kGN);
constexpr uint32_t kGTmemCols = kGN;
constexpr int kAttnThreads = 256;
// query rows (tokens x query heads of one kv head) per CTA: 64, or 128 with 64-dim heads when
// the chunk gives every SM three such CTAs (8 rows per thread: a larger register tile and
// half the K/V page loads per query; 8192-token prompt in 2048-token chunks 158.7 -> 146.0
// ms, while 512-1408-token prompts, too short to fill the SMs with 128-row CTAs, lost 1-3 %)
constexpr int kAttnRowsMin = 64;
constexpr int kAttnRowsWide = 128;

// error word of the handle: [0] code, [4] abort flag (the decode kernel's layout)
constexpr uint32_t kErrPrefillWait = 7;

enum Epi { EPI_QKV = 0, EPI_RESID = 1, EPI_SWIGLU = 2 };

struct GemmArgs {
  int T, K, n_tiles;
  // EPI_RESID: X[t][n*128 + j] += D[t][j]
  float* X;
  int ldx;
  // EPI_QKV: tiles [0, nq) are queries, [nq, nq + nk) keys, then values
  float* Q;
  uint16_t* kv;
  const int* pt;  // the slot's page table row
  const float2* rope;
  int nq, nk, layer, pos0, d, qdim, PL, Hkv, n_phys_pages, kv_fp16;
  // EPI_SWIGLU
  uint16_t* Ahi;
  uint16_t* Alo;
  int F;
  uint32_t* err;
  unsigned long long limit_ns;
};

__device__ __forceinline__ bool pf_aborted(const uint32_t* err) { return ld_relaxed_u32(err + 4) != 0; }

__device__ __forceinline__ void pf_fail(uint32_t* err, uint32_t where) {
  atomicCAS(err, 0u, kErrPrefillWait);
  atomicCAS(err + 3, 0u, where);
  atomicExch(err + 4, 1u);
}

// Bounded mbarrier wait: false on timeout (error recorded) or when another CTA aborted.
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, uint32_t* err,
                                        unsigned long long limit_ns, uint32_t where) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255) == 0) {
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      if (pf_aborted(err)) return false;
      if (now - t0 > limit_ns) {
        pf_fail(err, where);
        return false;
      }
    }
  }
}

__device__ __forceinline__ uint16_t kv_round(float v, int fp16) {
  return fp16 ? __half_as_ushort(__float2half_rn(v)) : __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

template <int EPI>
__global__ void __launch_bounds__(kGThreads, 1)
    pf_gemm(const __grid_constant__ CUtensorMap a_hi, const __grid_constant__ CUtensorMap a_lo,
            const __grid_constant__ CUtensorMap b0, const __grid_constant__ CUtensorMap b1,
            const __grid_constant__ CUtensorMap b2, const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kGStageBytes);
  uint64_t* empty = full + kGStages;
  uint64_t* accf = empty + kGStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accf + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kGM, n = blockIdx.y;
  const int nk = g.K / kGK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, kGTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {  // TMA producer
      const uint64_t pol = l2_evict_last_policy();  // tiles are read again by neighbouring CTAs
      int it = 0;
      for (; it < nk; ++it) {
        const int s = it % kGStages, use = it / kGStages;
        if (!pf_wait(&empty[s], (use & 1) ^ 1, g.err, g.limit_ns, 1)) break;
        uint8_t* st = smem + s * kGStageBytes;
        mbar_arrive_expect_tx(&full[s], kGStageBytes);
        tma_load_2d(st, &a_hi, it * kGK, m0, &full[s], pol);
        tma_load_2d(st + kGTile, &a_lo, it * kGK, m0, &full[s], pol);
        if constexpr (EPI == EPI_QKV) {
          const CUtensorMap* m = n < g.nq ? &b0 : n < g.nq + g.nk ? &b1 : &b2;
          const int r0 = (n < g.nq ? n : n < g.nq + g.nk ? n - g.nq : n - g.nq - g.nk) * kGN;
          tma_load_2d(st + 2 * kGTile, m, it * kGK, r0, &full[s], pol);
        } else if constexpr (EPI == EPI_SWIGLU) {  // 64 gate rows, then the same 64 up rows
          tma_load_2d(st + 2 * kGTile, &b0, it * kGK, n * (kGN / 2), &full[s], pol);
          tma_load_2d(st + 2 * kGTile + kGTile / 2, &b1, it * kGK, n * (kGN / 2), &full[s], pol);
        } else {
          tma_load_2d(st + 2 * kGTile, &b0, it * kGK, n * kGN, &full[s], pol);
        }
      }
      // every load issued lands before the CTA exits
      for (int q = it > kGStages ? it - kGStages : 0; q < it; ++q)
        if (!pf_wait(&full[q % kGStages], (q / kGStages) & 1, g.err, g.limit_ns, 2)) break;
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      for (int it = 0; it < nk; ++it) {
        const int s = it % kGStages, use = it / kGStages;
        if (!pf_wait(&full[s], use & 1, g.err, g.limit_ns, 3)) break;
        tc_fence_after();
        const uint32_t ah = smem_u32(smem + s * kGStageBytes), al = ah + kGTile, b = ah + 2 * kGTile;
#pragma unroll
        for (int j = 0; j < kGK / 16; ++j) {
          umma_f16(tmem, sw128_desc(ah + 32 * j), sw128_desc(b + 32 * j), kGIdesc, (it | j) != 0 ? 1u : 0u);
          umma_f16(tmem, sw128_desc(al + 32 * j), sw128_desc(b + 32 * j), kGIdesc, 1u);
        }
        umma_commit(&empty[s]);  // the stage is free once these MMAs have read it
      }
      umma_commit(accf);  // every MMA above has completed (also on an early exit)
    }
  } else {  // epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31
    const int q = warp & 3;
    const int row = m0 + 32 * q + lane;
    const bool valid = row < g.T;
    const uint32_t tb = tmem + ((uint32_t)(32 * q) << 16);
    // warp-uniform: the tensor-memory loads below are warp-collective
    const bool ok = __all_sync(0xFFFFFFFFu, pf_wait(accf, 0, g.err, g.limit_ns, 4));
    tc_fence_after();
    if (ok) {
      if constexpr (EPI == EPI_RESID) {
        for (int c0 = 0; c0 < kGN; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tb + (uint32_t)c0, r);
          tmem_ld_wait();
          if (valid) {
            float* x = g.X + (size_t)row * g.ldx + (size_t)n * kGN + c0;
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              float4 v = *reinterpret_cast<float4*>(x + j);
              v.x += __uint_as_float(r[j]);
              v.y += __uint_as_float(r[j + 1]);
              v.z += __uint_as_float(r[j + 2]);
              v.w += __uint_as_float(r[j + 3]);
              *reinterpret_cast<float4*>(x + j) = v;
            }
          }
        }
      } else if constexpr (EPI == EPI_SWIGLU) {
        for (int c0 = 0; c0 < kGN / 2; c0 += 32) {
          uint32_t gt[32], up[32];
          tmem_ld32(tb + (uint32_t)c0, gt);
          tmem_ld32(tb + (uint32_t)(kGN / 2 + c0), up);
          tmem_ld_wait();
          if (valid) {
            const size_t o = (size_t)row * g.F + (size_t)n * (kGN / 2) + c0;
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              uint16_t hi[8], lo[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float gv = __uint_as_float(gt[j + e]), uv = __uint_as_float(up[j + e]);
                split_bf16(gv / (1.0f + __expf(-gv)) * uv, hi[e], lo[e]);
              }
              *reinterpret_cast<uint4*>(g.Ahi + o + j) = *reinterpret_cast<const uint4*>(hi);
              *reinterpret_cast<uint4*>(g.Alo + o + j) = *reinterpret_cast<const uint4*>(lo);
            }
          }
        }
      } else {  // EPI_QKV
        const int sec = n < g.nq ? 0 : n < g.nq + g.nk ? 1 : 2;
        const int f0 = (sec == 0 ? n : sec == 1 ? n - g.nq : n - g.nq - g.nk) * kGN;
        const int d = g.d, half = d / 2;
        const int pos = g.pos0 + row;
        // pair groups of 32 frequencies: columns c + i0 + j and c + half + i0 + j
        for (int c = 0; c < kGN; c += d) {
          for (int i0 = 0; i0 < half; i0 += 32) {
            uint32_t x1[32], x2[32];
            tmem_ld32(tb + (uint32_t)(c + i0), x1);
            tmem_ld32(tb + (uint32_t)(c + half + i0), x2);
            tmem_ld_wait();
            if (!valid) continue;
            const int head = (f0 + c) / d;
            const float2* cs = g.rope + (size_t)pos * half + i0;
            if (sec == 0) {
              float* qq = g.Q + (size_t)row * g.qdim + (size_t)head * d + i0;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float a = __uint_as_float(x1[j]), b = __uint_as_float(x2[j]);
                const float2 r = cs[j];
                qq[j] = a * r.x - b * r.y;
                qq[j + half] = b * r.x + a * r.y;
              }
            } else {
              const int phys = g.pt[pos / g.PL];
              uint16_t* dst = g.kv + ((((size_t)g.layer * g.n_phys_pages + phys) * g.Hkv + head) * 2 + (sec - 1)) *
                                         (size_t)(g.PL * d) +
                              (size_t)(pos % g.PL) * d + i0;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                float a = __uint_as_float(x1[j]), b = __uint_as_float(x2[j]);
                if (sec == 1) {
                  const float2 r = cs[j];
                  const float ra = a * r.x - b * r.y, rb = b * r.x + a * r.y;
                  a = ra;
                  b = rb;
                }
                dst[j] = kv_round(a, g.kv_fp16);
                dst[j + half] = kv_round(b, g.kv_fp16);
              }
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kGTmemCols);
}

// X[t] = E[tok[t]] (bf16 -> fp32)
__global__ void pf_embed(const uint16_t* __restrict__ E, const int* __restrict__ tok, int T, int H,
                         float* __restrict__ X) {
  const int nch = H / 8;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < (long long)T * nch;
       e += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(e / nch), c = (int)(e % nch);
    const uint4 w = ldnc16(E + (size_t)tok[t] * H + c * 8);
    float4* x = reinterpret_cast<float4*>(X + (size_t)t * H + c * 8);
    x[0] = make_float4(bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
    x[1] = make_float4(bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w));
  }
}

// n = x / sqrt(mean(x^2) + eps) * g, one warp per token row, as bf16 high and low parts
__global__ void pf_norm_split(const float* __restrict__ X, int T, int H, const uint16_t* __restrict__ gain,
                              float eps, uint16_t* __restrict__ hi, uint16_t* __restrict__ lo) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= T) return;
  const float* x = X + (size_t)row * H;
  float ss = 0.f;
  for (int c = lane; c < H / 4; c += 32) {
    const float4 v = reinterpret_cast<const float4*>(x)[c];
    ss = fmaf(v.x, v.x, ss);
    ss = fmaf(v.y, v.y, ss);
    ss = fmaf(v.z, v.z, ss);
    ss = fmaf(v.w, v.w, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
  const float r = 1.0f / sqrtf(ss / (float)H + eps);
  for (int c = lane; c < H / 8; c += 32) {
    const float4 a = reinterpret_cast<const float4*>(x)[2 * c], b = reinterpret_cast<const float4*>(x)[2 * c + 1];
    const uint4 gw = ldnc16(gain + c * 8);
    const float v[8] = {a.x * bf_lo(gw.x), a.y * bf_hi(gw.x), a.z * bf_lo(gw.y), a.w * bf_hi(gw.y),
                        b.x * bf_lo(gw.z), b.y * bf_hi(gw.z), b.z * bf_lo(gw.w), b.w * bf_hi(gw.w)};
    uint16_t h8[8], l8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) split_bf16(v[e] * r, h8[e], l8[e]);
    *reinterpret_cast<uint4*>(hi + (size_t)row * H + c * 8) = *reinterpret_cast<const uint4*>(h8);
    *reinterpret_cast<uint4*>(lo + (size_t)row * H + c * 8) = *reinterpret_cast<const uint4*>(l8);
  }
}

template <bool F16>
__device__ __forceinline__ float kv_elem(uint4 w, int e) {
  const uint32_t u = e < 2 ? w.x : e < 4 ? w.y : e < 6 ? w.z : w.w;
  return (e & 1) ? kv_hi<F16>(u) : kv_lo<F16>(u);
}

// Causal GQA attention of a chunk's queries over the cache.  CTA = (kv head g,
// block of 64 / rep tokens, the last block first: blocks read more pages the later
// their tokens, so the longest go out first and the short ones fill the tail).  Its
// 64 query rows are the rep query heads of g for
// each token (row r: head g * rep + r / QB, token t0 + r % QB).  The KV pages of
// positions 0 .. the block's last position are read in order; per page the
// scores of every (row, position) pair, the running max / sum / output of an
// online softmax per row, and the key mask pos_key <= pos_query.  Thread (ty, tx)
// owns rows 4 ty .. 4 ty + 3 and keys tx * KPT .. (scores) or output dims
// tx * DPT .. (P V).  Output: o / l as bf16 high and low parts [T][qdim].
template <int DH, bool KV16F, int ROWS>
__global__ void __launch_bounds__(kAttnThreads)
    pf_attn(const float* __restrict__ Q, int T, int qdim, const uint16_t* __restrict__ kv, const int* __restrict__ pt,
            int layer, int n_phys_pages, int Hkv, int rep, int pos0, uint16_t* __restrict__ Ohi,
            uint16_t* __restrict__ Olo) {
  constexpr int PL = 16384 / (4 * DH);  // positions per KV page
  constexpr int KPT = PL / 16;          // keys per thread
  constexpr int DPT = DH / 16;          // output dims per thread
  constexpr int PSTR = PL + 4;          // padded row of the probabilities
  constexpr int RPT = ROWS / 16;        // query rows per thread
  extern __shared__ float sm[];
  float* qT = sm;                       // [DH][ROWS]
  float* kT = qT + DH * ROWS;           // [DH][PL]
  float* Vs = kT + DH * PL;             // [PL][DH]
  float* Ps = Vs + PL * DH;             // [ROWS][PSTR]
  const int QB = ROWS / rep;
  const int g = blockIdx.x, t0 = (gridDim.y - 1 - blockIdx.y) * QB;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  for (int e = tid; e < ROWS * DH; e += kAttnThreads) {
    const int r = e / DH, dd = e % DH, t = t0 + r % QB;
    qT[dd * ROWS + r] = t < T ? Q[(size_t)t * qdim + (size_t)(g * rep + r / QB) * DH + dd] : 0.f;
  }
  int qpos[RPT];
  bool rv[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int r = RPT * ty + i, t = t0 + r % QB;
    rv[i] = t < T;
    qpos[i] = pos0 + t;
  }
  float m[RPT], l[RPT];
  float2 o[RPT][DPT / 2];  // output dims in pairs (FFMA2)
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int e = 0; e < DPT / 2; ++e) o[i][e] = make_float2(0.f, 0.f);
  }
  const int last_pos = pos0 + min(T, t0 + QB) - 1;
  const int npages = last_pos / PL + 1;
  const float scale = 1.0f / sqrtf((float)DH);
  for (int pg = 0; pg < npages; ++pg) {
    __syncthreads();  // the previous page's reads are done
    const uint16_t* kp = kv + (((size_t)layer * n_phys_pages + pt[pg]) * Hkv + g) * (size_t)(2 * PL * DH);
    const uint16_t* vp = kp + PL * DH;
    for (int e = tid; e < PL * DH / 8; e += kAttnThreads) {  // K transposed: position fastest
      const int pos = e % PL, c = e / PL;
      const uint4 w = ldnc16(kp + (size_t)pos * DH + c * 8);
#pragma unroll
      for (int j = 0; j < 8; ++j) kT[(c * 8 + j) * PL + pos] = kv_elem<KV16F>(w, j);
    }
    for (int e = tid; e < PL * DH / 8; e += kAttnThreads) {  // V as is: dims fastest
      const int pos = e / (DH / 8), c = e % (DH / 8);
      const uint4 w = ldnc16(vp + (size_t)pos * DH + c * 8);
#pragma unroll
      for (int j = 0; j < 8; ++j) Vs[pos * DH + c * 8 + j] = kv_elem<KV16F>(w, j);
    }
    __syncthreads();
    // scores: packed FP32 FMA (FFMA2) over pairs of keys; each element rounds as fmaf
    float2 s2[RPT][KPT / 2];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
      for (int j = 0; j < KPT / 2; ++j) s2[i][j] = make_float2(0.f, 0.f);
#pragma unroll 8
    for (int dd = 0; dd < DH; ++dd) {
      float qa[RPT];
#pragma unroll
      for (int i = 0; i < RPT; i += 4) {
        const float4 qv = *reinterpret_cast<const float4*>(qT + dd * ROWS + RPT * ty + i);
        qa[i] = qv.x; qa[i + 1] = qv.y; qa[i + 2] = qv.z; qa[i + 3] = qv.w;
      }
      float2 kk[KPT / 2];
      if constexpr (KPT == 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(kT + dd * PL + 4 * tx);
        kk[0] = make_float2(k4.x, k4.y);
        kk[1] = make_float2(k4.z, k4.w);
      } else {
        kk[0] = *reinterpret_cast<const float2*>(kT + dd * PL + 2 * tx);
      }
#pragma unroll
      for (int i = 0; i < RPT; ++i)
#pragma unroll
        for (int j = 0; j < KPT / 2; ++j) s2[i][j] = __ffma2_rn(make_float2(qa[i], qa[i]), kk[j], s2[i][j]);
    }
    float s[RPT][KPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
      for (int j = 0; j < KPT / 2; ++j) {
        s[i][2 * j] = s2[i][j].x;
        s[i][2 * j + 1] = s2[i][j].y;
      }
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < KPT; ++j) {
        const int kpos = pg * PL + tx * KPT + j;
        s[i][j] = (rv[i] && kpos <= qpos[i]) ? s[i][j] * scale : -INFINITY;
        mx = fmaxf(mx, s[i][j]);
      }
#pragma unroll
      for (int off = 1; off < 16; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
      const float mn = fmaxf(m[i], mx);
      const float corr = mn == -INFINITY ? 1.f : __expf(m[i] - mn);
      float ps = 0.f;
#pragma unroll
      for (int j = 0; j < KPT; ++j) {
        const float p = mn == -INFINITY ? 0.f : __expf(s[i][j] - mn);
        Ps[(RPT * ty + i) * PSTR + tx * KPT + j] = p;
        ps += p;
      }
#pragma unroll
      for (int off = 1; off < 16; off <<= 1) ps += __shfl_xor_sync(0xFFFFFFFFu, ps, off);
      l[i] = l[i] * corr + ps;
      m[i] = mn;
#pragma unroll
      for (int e = 0; e < DPT / 2; ++e) {
        o[i][e].x *= corr;
        o[i][e].y *= corr;
      }
    }
    __syncthreads();
    // P.V, four keys per step: each row's four probabilities in one 16-byte load
    static_assert(PL % 4 == 0 && PSTR % 4 == 0, "float4 rows of probabilities");
#pragma unroll 2
    for (int k0 = 0; k0 < PL; k0 += 4) {
      float4 p4[RPT];
#pragma unroll
      for (int i = 0; i < RPT; ++i) p4[i] = *reinterpret_cast<const float4*>(Ps + (RPT * ty + i) * PSTR + k0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int k = k0 + kk;
        float2 v[DPT / 2];
#pragma unroll
        for (int e = 0; e < DPT / 2; e += 2) {
          const float4 v4 = *reinterpret_cast<const float4*>(Vs + k * DH + tx * DPT + 2 * e);
          v[e] = make_float2(v4.x, v4.y);
          v[e + 1] = make_float2(v4.z, v4.w);
        }
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
          const float pk = kk == 0 ? p4[i].x : kk == 1 ? p4[i].y : kk == 2 ? p4[i].z : p4[i].w;
#pragma unroll
          for (int e = 0; e < DPT / 2; ++e) o[i][e] = __ffma2_rn(make_float2(pk, pk), v[e], o[i][e]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    if (!rv[i]) continue;
    const int r = RPT * ty + i, t = t0 + r % QB;
    const float inv = 1.0f / l[i];
    const size_t base = (size_t)t * qdim + (size_t)(g * rep + r / QB) * DH + tx * DPT;
    uint16_t h[DPT], lo[DPT];
#pragma unroll
    for (int e = 0; e < DPT / 2; ++e) {
      split_bf16(o[i][e].x * inv, h[2 * e], lo[2 * e]);
      split_bf16(o[i][e].y * inv, h[2 * e + 1], lo[2 * e + 1]);
    }
#pragma unroll
    for (int e = 0; e < DPT; e += 4) {
      *reinterpret_cast<uint2*>(Ohi + base + e) = *reinterpret_cast<const uint2*>(h + e);
      *reinterpret_cast<uint2*>(Olo + base + e) = *reinterpret_cast<const uint2*>(lo + e);
    }
  }
}

// Causal GQA attention of a chunk's queries on the tensor cores (64-dim heads, bf16
// cache).  CTA = (kv head g, block of 128 / rep tokens, the last block first): its 128
// query rows are the rep query heads of g for each token (row r: head g * rep + r / QB,
// token t0 + r % QB), one row per tensor-memory lane.  Per KV page (64 positions):
//   - the 128 threads (one per query row) stage K as the B operand of S (64 key rows
//     of 64 dims, 128-byte swizzle) and V transposed as the B operand of P.V (64 dim
//     rows of 64 keys);
//   - thread 0 issues S = Q_hi K^T + Q_lo K^T (M = 128, N = 64, K = 64: 8 MMAs) into
//     tensor-memory columns 0..63 and commits;
//   - each thread reads its row of S back, applies the causal mask, updates the row's
//     online softmax (max m, sum l), rescales the row's output (kept in registers) and
//     writes P as bf16 high and low parts (the A operand);
//   - thread 0 issues P.V = P_hi V + P_lo V into columns 64..127 and commits, and every
//     thread adds it to its row's output.
// Two CTAs share an SM (one's loads overlap the other's MMAs and softmax).
// Q and P are split into bf16 high and low parts, so the products keep fp32-level
// accuracy; K and V are the cache's bf16 values.  Output: o / l as bf16 high and low
// parts [T][qdim].  Every wait is bounded (pf_wait); tensor memory is freed on every
// exit path.
constexpr int kTcAttnRows = 128;
constexpr int kTcAttnThreads = 128;  // one thread per query row; two CTAs per SM
constexpr int kTcAttnCols = 128;  // S in columns 0..63, P.V in 64..127
constexpr uint32_t kTcAttnIdesc = idesc_bf16(128, 64);
constexpr int kTcAttnSmem = 1024 + 2 * 16384 + 8192 + 8192 + 2 * 16384 + 64;

// byte offset of element (row, col) in a tile of 128-byte rows (64 bf16), 128-byte swizzle
__device__ __forceinline__ uint32_t sw128_off(int row, int col) {
  return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((((col >> 3) ^ (row & 7)) & 7) << 4) + (col & 7) * 2);
}

__global__ void __launch_bounds__(kTcAttnThreads, 2)
    pf_attn_tc(const float* __restrict__ Q, int T, int qdim, const uint16_t* __restrict__ kv,
               const int* __restrict__ pt, int layer, int n_phys_pages, int Hkv, int rep, int pos0,
               uint16_t* __restrict__ Ohi, uint16_t* __restrict__ Olo, uint32_t* err, unsigned long long limit_ns) {
  constexpr int DH = 64, PL = 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* qhi = smem;                // [128][64] bf16, swizzled
  uint8_t* qlo = qhi + 16384;
  uint8_t* kt = qlo + 16384;          // [64 keys][64 dims]
  uint8_t* vt = kt + 8192;            // [64 dims][64 keys]
  uint8_t* phi = vt + 8192;           // [128][64 keys]
  uint8_t* plo = phi + 16384;
  uint64_t* sdone = reinterpret_cast<uint64_t*>(plo + 16384);
  uint64_t* pvdone = sdone + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(pvdone + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int QB = kTcAttnRows / rep;
  const int g = blockIdx.x, t0 = (gridDim.y - 1 - blockIdx.y) * QB;

  if (tid == 0) {
    mbar_init(sdone, 1);
    mbar_init(pvdone, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, kTcAttnCols);
  // queries, scaled by 1/sqrt(d), as bf16 high and low parts (the A operand of S)
  const float scale = 1.0f / sqrtf((float)DH);
  for (int e = tid; e < kTcAttnRows * (DH / 8); e += kTcAttnThreads) {
    const int r = e / (DH / 8), c = e % (DH / 8), t = t0 + r % QB;
    uint16_t h8[8], l8[8];
    if (t < T) {
      const float* src = Q + (size_t)t * qdim + (size_t)(g * rep + r / QB) * DH + c * 8;
      const float4 a = *reinterpret_cast<const float4*>(src), b = *reinterpret_cast<const float4*>(src + 4);
      const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) split_bf16(v[j] * scale, h8[j], l8[j]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) h8[j] = l8[j] = 0;
    }
    *reinterpret_cast<uint4*>(qhi + sw128_off(r, c * 8)) = *reinterpret_cast<const uint4*>(h8);
    *reinterpret_cast<uint4*>(qlo + sw128_off(r, c * 8)) = *reinterpret_cast<const uint4*>(l8);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  // this thread's query row (tensor-memory lane = row = thread)
  const int row = tid;                 // meaningful for tid < 128
  const int qt = t0 + row % QB;
  const bool rv = tid < kTcAttnRows && qt < T;
  const int qpos = pos0 + qt;
  float m = -INFINITY, l = 0.f, o[DH];
#pragma unroll
  for (int d = 0; d < DH; ++d) o[d] = 0.f;
  const int last_pos = pos0 + min(T, t0 + QB) - 1;
  const int npages = last_pos / PL + 1;
  const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  bool ok = true;
  for (int pg = 0; pg < npages; ++pg) {
    // K as is (key rows), V transposed (dim rows), both swizzled
    const uint16_t* kp = kv + (((size_t)layer * n_phys_pages + pt[pg]) * Hkv + g) * (size_t)(2 * PL * DH);
    const uint16_t* vp = kp + PL * DH;
    for (int e = tid; e < PL * (DH / 8); e += kTcAttnThreads) {
      const int r = e / (DH / 8), c = e % (DH / 8);
      const uint4 w = ldnc16(kp + (size_t)r * DH + c * 8);
      *reinterpret_cast<uint4*>(kt + sw128_off(r, c * 8)) = w;
      const uint4 v = ldnc16(vp + (size_t)r * DH + c * 8);
      const uint16_t* v16 = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
      for (int j = 0; j < 8; ++j) *reinterpret_cast<uint16_t*>(vt + sw128_off(c * 8 + j, r)) = v16[j];
    }
    fence_proxy_async_smem();  // the tensor cores read the tiles through the async proxy
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0 && ok) {
      const uint32_t a0 = smem_u32(qhi), a1 = smem_u32(qlo), b = smem_u32(kt);
#pragma unroll
      for (int j = 0; j < DH / 16; ++j) {
        umma_f16(tmem, sw128_desc(a0 + 32 * j), sw128_desc(b + 32 * j), kTcAttnIdesc, j ? 1u : 0u);
        umma_f16(tmem, sw128_desc(a1 + 32 * j), sw128_desc(b + 32 * j), kTcAttnIdesc, 1u);
      }
      umma_commit(sdone);
    }
    if (warp < 4) {  // every warp (128 threads): one query row per thread
      ok = __all_sync(0xFFFFFFFFu, ok && pf_wait(sdone, pg & 1, err, limit_ns, 11));
      tc_fence_after();
      float sv[PL];
      if (ok) {
#pragma unroll
        for (int c0 = 0; c0 < PL; c0 += 32) {
          uint32_t r32[32];
          tmem_ld32(tl + (uint32_t)c0, r32);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) sv[c0 + j] = __uint_as_float(r32[j]);
        }
      }
      // online softmax of this row over the page's positions (key pos <= query pos)
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < PL; ++c) {
        const int kpos = pg * PL + c;
        sv[c] = (rv && kpos <= qpos) ? sv[c] : -INFINITY;
        mx = fmaxf(mx, sv[c]);
      }
      const float mn = fmaxf(m, mx);
      const float corr = mn == -INFINITY ? 1.f : __expf(m - mn);
      float ps = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < PL; c0 += 8) {
        uint16_t h8[8], l8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float pv = mn == -INFINITY ? 0.f : __expf(sv[c0 + j] - mn);
          ps += pv;
          split_bf16(pv, h8[j], l8[j]);
        }
        *reinterpret_cast<uint4*>(phi + sw128_off(row, c0)) = *reinterpret_cast<const uint4*>(h8);
        *reinterpret_cast<uint4*>(plo + sw128_off(row, c0)) = *reinterpret_cast<const uint4*>(l8);
      }
      l = l * corr + ps;
      m = mn;
#pragma unroll
      for (int d = 0; d < DH; ++d) o[d] *= corr;
      fence_proxy_async_smem();
      tc_fence_before();
      asm volatile("bar.sync 1, 128;" ::: "memory");  // every row's P is written
      tc_fence_after();
      if (tid == 0 && ok) {
        const uint32_t a0 = smem_u32(phi), a1 = smem_u32(plo), b = smem_u32(vt);
#pragma unroll
        for (int j = 0; j < PL / 16; ++j) {
          umma_f16(tmem + 64u, sw128_desc(a0 + 32 * j), sw128_desc(b + 32 * j), kTcAttnIdesc, j ? 1u : 0u);
          umma_f16(tmem + 64u, sw128_desc(a1 + 32 * j), sw128_desc(b + 32 * j), kTcAttnIdesc, 1u);
        }
        umma_commit(pvdone);
      }
      ok = __all_sync(0xFFFFFFFFu, ok && pf_wait(pvdone, pg & 1, err, limit_ns, 12));
      tc_fence_after();
      if (ok) {
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 32) {
          uint32_t r32[32];
          tmem_ld32(tl + 64u + (uint32_t)c0, r32);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[c0 + j] += __uint_as_float(r32[j]);
        }
      }
    }
    // the tiles are free once P.V has read them (every thread saw it complete)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
    if (!ok) break;
  }
  if (rv && ok) {
    const int t = qt, h = g * rep + row / QB;
    const float inv = 1.0f / l;
    uint16_t* dh = Ohi + (size_t)t * qdim + (size_t)h * DH;
    uint16_t* dl = Olo + (size_t)t * qdim + (size_t)h * DH;
#pragma unroll
    for (int d0 = 0; d0 < DH; d0 += 8) {
      uint16_t h8[8], l8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) split_bf16(o[d0 + j] * inv, h8[j], l8[j]);
      *reinterpret_cast<uint4*>(dh + d0) = *reinterpret_cast<const uint4*>(h8);
      *reinterpret_cast<uint4*>(dl + d0) = *reinterpret_cast<const uint4*>(l8);
    }
  }
  // every MMA issued has completed (each was waited for) before tensor memory is freed
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTcAttnCols);
}

template <int DH, int ROWS>
constexpr int attn_smem() {
  return (DH * ROWS + DH * (16384 / (4 * DH)) * 2 + ROWS * (16384 / (4 * DH) + 4)) * 4;
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_pf_mutex;
EncodeTiled g_pf_encode = nullptr;

// bf16 [rows][inner] row-major, boxes of 64 x box_rows, 128-byte swizzle, zero fill
bool encode(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kGK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  std::memset(m, 0, sizeof *m);
  return g_pf_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

struct PrefillPlan {
  Dims D{};
  int chunk = 0;
  int n_sm = 148;  // SMs of the device (the attention's tile choice)
  const uint16_t* embed = nullptr;
  std::vector<const uint16_t*> attn_norm, mlp_norm;
  std::vector<CUtensorMap> wq, wk, wv, wo, wg, wu, wd;
  float* X = nullptr;
  float* Q = nullptr;
  uint16_t *Nhi = nullptr, *Nlo = nullptr, *Ohi = nullptr, *Olo = nullptr, *Ahi = nullptr, *Alo = nullptr;
  std::vector<void*> allocs;
};

bool prefill_supported(const Dims& D) {
  return D.H % kGN == 0 && D.qdim % kGN == 0 && D.kvdim % kGN == 0 && D.F % (kGN / 2) == 0 &&
         (D.d == 64 || D.d == 128) && kAttnRowsMin % D.rep == 0;
}

void prefill_destroy(PrefillPlan* p) {
  if (!p) return;
  for (void* a : p->allocs) cudaFree(a);
  delete p;
}

mk_status prefill_create(const Dims& D, const mk_weights* w, int chunk, PrefillPlan** out) {
  *out = nullptr;
  if (!prefill_supported(D) || chunk < 1) return MK_ERR_UNSUPPORTED;
  int dev = 0, n_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm < 1)
    return MK_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(g_pf_mutex);
    if (!g_pf_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess || !fn ||
          q != cudaDriverEntryPointSuccess)
        return MK_ERR_CUDA;
      g_pf_encode = reinterpret_cast<EncodeTiled>(fn);
    }
  }
  PrefillPlan* p = new PrefillPlan();
  p->n_sm = n_sm;
  p->D = D;
  p->chunk = chunk;
  p->embed = static_cast<const uint16_t*>(w->embed);
  bool ok = true;
  for (int l = 0; l < D.L && ok; ++l) {
    p->attn_norm.push_back(static_cast<const uint16_t*>(w->attn_norm[l]));
    p->mlp_norm.push_back(static_cast<const uint16_t*>(w->mlp_norm[l]));
    CUtensorMap m;
    ok &= encode(&m, w->wq[l], D.H, D.qdim, kGN); p->wq.push_back(m);
    ok &= encode(&m, w->wk[l], D.H, D.kvdim, kGN); p->wk.push_back(m);
    ok &= encode(&m, w->wv[l], D.H, D.kvdim, kGN); p->wv.push_back(m);
    ok &= encode(&m, w->wo[l], D.qdim, D.H, kGN); p->wo.push_back(m);
    ok &= encode(&m, w->w_gate[l], D.H, D.F, kGN / 2); p->wg.push_back(m);
    ok &= encode(&m, w->w_up[l], D.H, D.F, kGN / 2); p->wu.push_back(m);
    ok &= encode(&m, w->w_down[l], D.F, D.H, kGN); p->wd.push_back(m);
  }
  auto alloc = [&](void** ptr, size_t bytes) {
    if (!ok) return;
    if (cudaMalloc(ptr, bytes) != cudaSuccess) { ok = false; *ptr = nullptr; return; }
    p->allocs.push_back(*ptr);
  };
  const size_t T = (size_t)chunk;
  alloc((void**)&p->X, T * D.H * 4);
  alloc((void**)&p->Q, T * D.qdim * 4);
  alloc((void**)&p->Nhi, T * D.H * 2);
  alloc((void**)&p->Nlo, T * D.H * 2);
  alloc((void**)&p->Ohi, T * D.qdim * 2);
  alloc((void**)&p->Olo, T * D.qdim * 2);
  alloc((void**)&p->Ahi, T * D.F * 2);
  alloc((void**)&p->Alo, T * D.F * 2);
  if (ok) {
    ok &= cudaFuncSetAttribute(pf_gemm<EPI_QKV>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pf_gemm<EPI_RESID>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pf_gemm<EPI_SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmem) ==
          cudaSuccess;
    ok &= cudaFuncSetAttribute(pf_attn<64, false, kAttnRowsMin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn_smem<64, kAttnRowsMin>()) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pf_attn<64, true, kAttnRowsMin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn_smem<64, kAttnRowsMin>()) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pf_attn<64, false, kAttnRowsWide>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn_smem<64, kAttnRowsWide>()) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pf_attn<64, true, kAttnRowsWide>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn_smem<64, kAttnRowsWide>()) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pf_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcAttnSmem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pf_attn<128, false, kAttnRowsMin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn_smem<128, kAttnRowsMin>()) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pf_attn<128, true, kAttnRowsMin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn_smem<128, kAttnRowsMin>()) == cudaSuccess;
  }
  if (!ok) {
    prefill_destroy(p);
    return MK_ERR_OOM;
  }
  *out = p;
  return MK_OK;
}

mk_status prefill_run(PrefillPlan* p, const PrefillCtx& c, const int* tokens_dev, int n, int slot, int pos0,
                      cudaStream_t st) {
  const Dims& D = p->D;
  const int* pt = c.page_table + (size_t)slot * D.pages_per_seq;
  for (int c0 = 0; c0 < n; c0 += p->chunk) {
    const int T = std::min(p->chunk, n - c0), pos = pos0 + c0;
    CUtensorMap nhi, nlo, ohi, olo, ahi, alo;
    if (!encode(&nhi, p->Nhi, D.H, T, kGM) || !encode(&nlo, p->Nlo, D.H, T, kGM) ||
        !encode(&ohi, p->Ohi, D.qdim, T, kGM) || !encode(&olo, p->Olo, D.qdim, T, kGM) ||
        !encode(&ahi, p->Ahi, D.F, T, kGM) || !encode(&alo, p->Alo, D.F, T, kGM))
      return MK_ERR_CUDA;
    GemmArgs g{};
    g.T = T;
    g.err = c.err_code;
    g.limit_ns = c.wait_limit_ns;
    const int mt = (T + kGM - 1) / kGM;
    pf_embed<<<(T * (D.H / 8) + 255) / 256, 256, 0, st>>>(p->embed, tokens_dev + c0, T, D.H, p->X);
    for (int l = 0; l < D.L; ++l) {
      pf_norm_split<<<(T + 7) / 8, 256, 0, st>>>(p->X, T, D.H, p->attn_norm[l], D.eps, p->Nhi, p->Nlo);
      GemmArgs q = g;
      q.K = D.H;
      q.Q = p->Q;
      q.kv = c.kv;
      q.pt = pt;
      q.rope = c.rope;
      q.nq = D.qdim / kGN;
      q.nk = D.kvdim / kGN;
      q.layer = l;
      q.pos0 = pos;
      q.d = D.d;
      q.qdim = D.qdim;
      q.PL = D.PL;
      q.Hkv = D.Hkv;
      q.n_phys_pages = D.n_phys_pages;
      q.kv_fp16 = D.kv_fp16;
      pf_gemm<EPI_QKV><<<dim3(mt, q.nq + 2 * q.nk), kGThreads, kGSmem, st>>>(nhi, nlo, p->wq[l], p->wk[l],
                                                                             p->wv[l], q);
      if (l == D.L - 1) break;  // only the last layer's K and V are read later
      // 128-row CTAs where the chunk gives every SM three of them (64-dim heads)
      const bool wide = D.d == 64 && (long long)((T + kAttnRowsWide / D.rep - 1) / (kAttnRowsWide / D.rep)) * D.Hkv >=
                                         3LL * p->n_sm;
      const int qb = (wide ? kAttnRowsWide : kAttnRowsMin) / D.rep;  // tokens per CTA
      const dim3 ag(D.Hkv, (T + qb - 1) / qb);
#define MK_PF_ATTN(DH_, F16_, ROWS_)                                                                      \
  pf_attn<DH_, F16_, ROWS_><<<ag, kAttnThreads, attn_smem<DH_, ROWS_>(), st>>>(                           \
      p->Q, T, D.qdim, c.kv, pt, l, D.n_phys_pages, D.Hkv, D.rep, pos, p->Ohi, p->Olo)
      if (D.d == 64 && !D.kv_fp16 && kTcAttnRows % D.rep == 0) {  // tensor cores
        const int qbt = kTcAttnRows / D.rep;
        pf_attn_tc<<<dim3(D.Hkv, (T + qbt - 1) / qbt), kTcAttnThreads, kTcAttnSmem, st>>>(
            p->Q, T, D.qdim, c.kv, pt, l, D.n_phys_pages, D.Hkv, D.rep, pos, p->Ohi, p->Olo, g.err, g.limit_ns);
      } else if (D.d == 64) {
        if (wide) {
          if (D.kv_fp16) MK_PF_ATTN(64, true, kAttnRowsWide);
          else MK_PF_ATTN(64, false, kAttnRowsWide);
        } else {
          if (D.kv_fp16) MK_PF_ATTN(64, true, kAttnRowsMin);
          else MK_PF_ATTN(64, false, kAttnRowsMin);
        }
      } else {
        if (D.kv_fp16) MK_PF_ATTN(128, true, kAttnRowsMin);
        else MK_PF_ATTN(128, false, kAttnRowsMin);
      }
#undef MK_PF_ATTN
      GemmArgs r = g;
      r.K = D.qdim;
      r.X = p->X;
      r.ldx = D.H;
      pf_gemm<EPI_RESID><<<dim3(mt, D.H / kGN), kGThreads, kGSmem, st>>>(ohi, olo, p->wo[l], p->wo[l], p->wo[l], r);
      pf_norm_split<<<(T + 7) / 8, 256, 0, st>>>(p->X, T, D.H, p->mlp_norm[l], D.eps, p->Nhi, p->Nlo);
      GemmArgs s = g;
      s.K = D.H;
      s.Ahi = p->Ahi;
      s.Alo = p->Alo;
      s.F = D.F;
      pf_gemm<EPI_SWIGLU><<<dim3(mt, D.F / (kGN / 2)), kGThreads, kGSmem, st>>>(nhi, nlo, p->wg[l], p->wu[l],
                                                                                p->wg[l], s);
      GemmArgs dn = g;
      dn.K = D.F;
      dn.X = p->X;
      dn.ldx = D.H;
      pf_gemm<EPI_RESID><<<dim3(mt, D.H / kGN), kGThreads, kGSmem, st>>>(ahi, alo, p->wd[l], p->wd[l], p->wd[l], dn);
    }
    if (cudaGetLastError() != cudaSuccess) return MK_ERR_CUDA;
  }
  return MK_OK;
}

}  // namespace mk
