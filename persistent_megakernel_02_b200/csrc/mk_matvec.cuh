// mk_matvec.cuh -- the CUDA-core matvec pieces shared by the decode kernel and
// the engine measurement (mk_engines.cu): the shared-memory ring position, the
// bf16 x fp32 page dot products, and the warp reduce-scatter.
#pragma once

#include "mk_device.cuh"

namespace mk {

// Position of a page in the ring protocol (see the kernel): its slot and the
// parity of the slot's use count, its full barrier and that barrier's parity.
// Advanced incrementally so the hot loops divide by the ring size only once.
struct RingPos {
  uint32_t slot, sphase, fidx, fphase;
  __device__ __forceinline__ void init(uint32_t page, uint32_t NP) {
    slot = page % NP;
    sphase = (page / NP) & 1u;
    fidx = page % (2 * NP);
    fphase = (page / (2 * NP)) & 1u;
  }
  __device__ __forceinline__ void advance(uint32_t n, uint32_t NP) {  // n <= NP
    slot += n;
    if (slot >= NP) { slot -= NP; sphase ^= 1u; }
    fidx += n;
    if (fidx >= 2 * NP) { fidx -= 2 * NP; fphase ^= 1u; }
  }
};

// acc[r][b] += W[r][k] * act[b][k] over this lane's 8-element chunks c = lane,
// lane + 32, ...; two partial sums per row (packed FP32 FMA, FFMA2).  The tile
// is RT rows of nch chunks in shared memory; act is staged in the split layout.
// Chunks not unrolled for 1-2 lanes (a Llama-3.2-1B batch-1 step measured 453 us,
// 456 unrolled by 2, 461 by 4: smaller code for the five inlined copies), by 4
// for more lanes.
template <int RT, int NBT>
__device__ __forceinline__ void mv_core(uint32_t tile, uint32_t alo, uint32_t ahi, int nch, int lane,
                                        float2 (&acc)[RT][NBT]) {
  constexpr int kUnroll = NBT <= 2 ? 1 : 4;
#pragma unroll kUnroll
  for (int c = lane; c < nch; c += 32) {
    float2 x[NBT][4];
#pragma unroll
    for (int b = 0; b < NBT; ++b) {
      const float4 l = lds128f(alo + (uint32_t)(b * nch + c) * 16u);
      const float4 h = lds128f(ahi + (uint32_t)(b * nch + c) * 16u);
      x[b][0] = make_float2(l.x, l.y);
      x[b][1] = make_float2(l.z, l.w);
      x[b][2] = make_float2(h.x, h.y);
      x[b][3] = make_float2(h.z, h.w);
    }
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const uint4 w = lds128(tile + (uint32_t)(r * nch + c) * 16u);
      const float2 w0 = make_float2(bf_lo(w.x), bf_hi(w.x)), w1 = make_float2(bf_lo(w.y), bf_hi(w.y));
      const float2 w2 = make_float2(bf_lo(w.z), bf_hi(w.z)), w3 = make_float2(bf_lo(w.w), bf_hi(w.w));
#pragma unroll
      for (int b = 0; b < NBT; ++b) {
        float2 s = acc[r][b];
        s = __ffma2_rn(w0, x[b][0], s);
        s = __ffma2_rn(w1, x[b][1], s);
        s = __ffma2_rn(w2, x[b][2], s);
        s = __ffma2_rn(w3, x[b][3], s);
        acc[r][b] = s;
      }
    }
  }
}

// Warp reduce-scatter of N per-lane values: while more than KEEP values remain,
// each lane keeps the half picked by its lane bit and adds its partner's copy of
// that half; the remaining lane bits are reduced in full.  Afterwards every lane
// holds rs_left(N, KEEP) totals, the first with index rs_base(N, KEEP, lane), and
// lanes that differ only in the bits of rs_dup_mask hold the same totals.
template <int N, int n, int KEEP, int O>
__device__ __forceinline__ void warp_rs(float (&v)[N], int lane) {
  if constexpr (O > 0) {
    if constexpr (n > KEEP) {
      const bool up = (lane & O) != 0;
#pragma unroll
      for (int i = 0; i < n / 2; ++i) {
        const float a = v[i], b = v[i + n / 2];
        v[i] = (up ? b : a) + __shfl_xor_sync(0xFFFFFFFFu, up ? a : b, O);
      }
      warp_rs<N, n / 2, KEEP, O / 2>(v, lane);
    } else {
#pragma unroll
      for (int i = 0; i < n; ++i) v[i] += __shfl_xor_sync(0xFFFFFFFFu, v[i], O);
      warp_rs<N, n, KEEP, O / 2>(v, lane);
    }
  }
}
__host__ __device__ constexpr int rs_left(int n, int keep) {
  for (int o = 16; o >= 1; o >>= 1)
    if (n > keep) n /= 2;
  return n;
}
__host__ __device__ constexpr int rs_dup_mask(int n, int keep) {
  int m = 0;
  for (int o = 16; o >= 1; o >>= 1) {
    if (n > keep) n /= 2;
    else m |= o;
  }
  return m;
}
__device__ __forceinline__ int rs_base(int n, int keep, int lane) {
  int idx = 0;
  for (int o = 16; o >= 1; o >>= 1)
    if (n > keep) {
      if (lane & o) idx += n / 2;
      n /= 2;
    }
  return idx;
}

}  // namespace mk
