// mk_noalloc.cu -- the greedy head (final RMSNorm, LM-head matvec, argmax) as a
// stand-alone call whose only working memory is a fixed static device array.
//
// This is the last stage of a decode step -- what the persistent kernel's LM-head
// instruction does -- offered to callers that run the decoder layers themselves
// and cannot allocate device memory on their call path: code inside a framework
// whose caching allocator already owns the GPU's memory (a raw cudaMalloc there
// can fail, or synchronise the whole device while it waits for memory), and
// latency-critical loops that forbid allocation once they have started.  It has
// no counterpart in the method this library implements; it is a convenience of
// the library.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "../../include/mk.h"
#include "mk_device.cuh"

namespace {

constexpr int kHeadThreads = 256;
constexpr int kHeadWarps = kHeadThreads / 32;
constexpr int kHeadMaxLanes = 8;
constexpr int kHeadMaxActFloats = 16384;  // lanes * hidden staged in shared memory
constexpr int kCounterBytes = 256;        // completion counter, at the start of the array
constexpr int kMaxBlocks = (MK_NOALLOC_SCRATCH_BYTES - kCounterBytes) / (kHeadMaxLanes * 8);

// The working memory of every call: [0, 256) the completion counter, then the
// best (value bits, index) of every block and lane.  Zero when the module loads;
// the last block of each call sets the counter back to zero.  Calls that overlap
// on the GPU share it and race.
static __device__ __align__(256) unsigned char g_head_scratch[MK_NOALLOC_SCRATCH_BYTES];

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

__global__ void __launch_bounds__(kHeadThreads) greedy_head_kernel(
    const float* __restrict__ hidden, int nb, int H, const uint16_t* __restrict__ gain,
    const uint16_t* __restrict__ W, int V, float eps, float* __restrict__ logits, int* __restrict__ ids,
    unsigned char* scratch) {
  extern __shared__ float hs[];  // normalised hidden state [nb][H]
  __shared__ float red[kHeadWarps][kHeadMaxLanes];
  __shared__ float bvs[kHeadWarps][kHeadMaxLanes];
  __shared__ int bis[kHeadWarps][kHeadMaxLanes];
  __shared__ int is_last;
  unsigned* counter = reinterpret_cast<unsigned*>(scratch);
  int2* part = reinterpret_cast<int2*>(scratch + kCounterBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // 1. RMSNorm of every lane's hidden state, gain applied, into shared memory
  for (int b = 0; b < nb; ++b) {
    float ss = 0.f;
    for (int k = tid; k < H; k += kHeadThreads) {
      const float v = hidden[(size_t)b * H + k];
      ss = fmaf(v, v, ss);
      hs[b * H + k] = v * mk::bf_lo((uint32_t)gain[k]);
    }
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if (lane == 0) red[warp][b] = ss;
  }
  __syncthreads();
  for (int b = 0; b < nb; ++b) {
    float t = 0.f;
    for (int w = 0; w < kHeadWarps; ++w) t += red[w][b];
    const float r = 1.0f / sqrtf(t / (float)H + eps);
    for (int k = tid; k < H; k += kHeadThreads) hs[b * H + k] *= r;
  }
  __syncthreads();

  // 2. one warp per LM-head row: logits and a running argmax per lane
  float bv[kHeadMaxLanes];
  int bi[kHeadMaxLanes];
#pragma unroll
  for (int b = 0; b < kHeadMaxLanes; ++b) { bv[b] = -INFINITY; bi[b] = 0x7FFFFFFF; }
  const int nch = H >> 3;
  for (int r = blockIdx.x * kHeadWarps + warp; r < V; r += gridDim.x * kHeadWarps) {
    float acc[kHeadMaxLanes];
#pragma unroll
    for (int b = 0; b < kHeadMaxLanes; ++b) acc[b] = 0.f;
    const uint16_t* row = W + (size_t)r * H;
    for (int c = lane; c < nch; c += 32) {
      const uint4 w = mk::ldnc16(row + c * 8);
      const float f[8] = {mk::bf_lo(w.x), mk::bf_hi(w.x), mk::bf_lo(w.y), mk::bf_hi(w.y),
                          mk::bf_lo(w.z), mk::bf_hi(w.z), mk::bf_lo(w.w), mk::bf_hi(w.w)};
#pragma unroll
      for (int b = 0; b < kHeadMaxLanes; ++b) {
        if (b >= nb) break;
        const float* hb = hs + b * H + c * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[b] = fmaf(f[e], hb[e], acc[b]);
      }
    }
#pragma unroll
    for (int b = 0; b < kHeadMaxLanes; ++b) {
      if (b >= nb) break;
      float s = acc[b];
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
      if (lane == 0 && logits) logits[(size_t)b * V + r] = s;
      if (better(s, r, bv[b], bi[b])) { bv[b] = s; bi[b] = r; }
    }
  }

  // 3. block best per lane into the scratch array; the last block reduces
  if (lane == 0)
    for (int b = 0; b < nb; ++b) { bvs[warp][b] = bv[b]; bis[warp][b] = bi[b]; }
  __syncthreads();
  if (tid < nb) {
    float v = -INFINITY;
    int i = 0x7FFFFFFF;
    for (int w = 0; w < kHeadWarps; ++w)
      if (better(bvs[w][tid], bis[w][tid], v, i)) { v = bvs[w][tid]; i = bis[w][tid]; }
    part[blockIdx.x * kHeadMaxLanes + tid] = make_int2(__float_as_int(v), i);
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    is_last = atomicAdd(counter, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (is_last) {
    __threadfence();
    if (tid < nb) {
      float v = -INFINITY;
      int i = 0x7FFFFFFF;
      for (int g = 0; g < (int)gridDim.x; ++g) {
        const int2 e = __ldcg(part + g * kHeadMaxLanes + tid);
        if (better(__int_as_float(e.x), e.y, v, i)) { v = __int_as_float(e.x); i = e.y; }
      }
      ids[tid] = (i >= 0 && i < V) ? i : 0;
    }
    if (tid == 0) *counter = 0u;  // the next call starts from zero
  }
}

// Device address of the static array, looked up once per device (with that
// device current) on the first call that runs there, together with the kernel's
// shared-memory attribute.  Both belong to the device's primary context: after a
// cudaDeviceReset the cached values are stale, so this entry point is not usable
// again in that process once its device has been reset.
std::mutex g_setup_mutex;
void* g_scratch_ptr[64];
int g_sm_count[64];

mk_status scratch_for_device(int dev, void** ptr, int* sms) {
  if (dev < 0 || dev >= 64) return MK_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_head_scratch) != cudaSuccess || !p) return MK_ERR_CUDA;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MK_ERR_CUDA;
    if (cudaFuncSetAttribute(greedy_head_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kHeadMaxActFloats * 4) != cudaSuccess)
      return MK_ERR_CUDA;
    g_sm_count[dev] = n;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  *sms = g_sm_count[dev];
  return MK_OK;
}

}  // namespace

extern "C" mk_status mk_greedy_head_noalloc(const float* hidden_dev, int32_t nb, int32_t hidden,
                                            const void* final_norm, const void* lm_head, int32_t vocab,
                                            float rms_eps, float* logits_dev, int32_t* ids_dev,
                                            void* stream) {
  if (!hidden_dev || !final_norm || !lm_head || !ids_dev) return MK_ERR_INVALID_ARG;
  if (nb < 1 || hidden < 8 || hidden % 8 || vocab < 1 || !(rms_eps >= 0.f) || !std::isfinite(rms_eps))
    return MK_ERR_INVALID_ARG;
  if (((uintptr_t)lm_head & 15u) != 0) return MK_ERR_INVALID_ARG;
  // beyond what the scratch array (8 lanes per block) and the shared-memory staging hold
  if (nb > kHeadMaxLanes || (long long)nb * hidden > kHeadMaxActFloats) return MK_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MK_ERR_CUDA;
  void* scratch = nullptr;
  int sms = 0;
  mk_status s = scratch_for_device(dev, &scratch, &sms);
  if (s != MK_OK) return s;
  const int rows_per_block = kHeadWarps;
  int blocks = (vocab + rows_per_block - 1) / rows_per_block;
  blocks = blocks < 4 * sms ? blocks : 4 * sms;
  if (blocks > kMaxBlocks) blocks = kMaxBlocks;
  const size_t smem = (size_t)nb * hidden * sizeof(float);
  // An error left pending by some earlier call of the caller's is not this call's
  // to report or to clear: refuse to launch and leave it in place.
  if (cudaPeekAtLastError() != cudaSuccess) return MK_ERR_CUDA;
  greedy_head_kernel<<<blocks, kHeadThreads, smem, (cudaStream_t)stream>>>(
      hidden_dev, nb, hidden, (const uint16_t*)final_norm, (const uint16_t*)lm_head, vocab, rms_eps,
      logits_dev, ids_dev, (unsigned char*)scratch);
  return cudaGetLastError() == cudaSuccess ? MK_OK : MK_ERR_CUDA;  // this launch's own error
}
