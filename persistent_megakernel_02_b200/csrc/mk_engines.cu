// mk_engines.cu -- the two engines a decode step's matvecs can run on, measured
// apart on the same streaming problem: Y[b][r] = sum_k W[r][k] X[b][k] for a
// bf16 weight matrix W [rows][K] in HBM and nb <= 8 fp32 activation rows.
//
//   engine 0  CUDA cores: the decode kernel's engine.  A producer thread
//             bulk-copies pages of whole rows into a shared-memory ring; each
//             consumer warp takes whole pages and runs the packed-FP32-FMA dot
//             products (mv_core), then a warp reduction.
//   engine 1  5th-generation tensor cores: TMA loads 128 x 64 bf16 tiles of W
//             (128-byte swizzle) into a ring; one thread issues tcgen05.mma
//             (M = 128 rows, N = 16, K = 16 per instruction) with the
//             activations as the B operand, split into bf16 high and low parts
//             (N columns 0-7 and 8-15) so the product keeps fp32-level accuracy;
//             the fp32 accumulators live in tensor memory, two buffers, read back
//             by four warps with tcgen05.ld.
//
// The Hazy megakernel article (section "Megakernel: a deep-fusion design from
// scratch") says tensor cores win again on Blackwell; this file is how that is
// checked per batch size rather than assumed.  Every wait is bounded; on
// timeout the kernels record an error and return.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "../../include/mk.h"
#include "mk_matvec.cuh"
#include "mk_plan.h"
#include "mk_tc.cuh"

namespace {

using namespace mk;

// error word of the last engine launch (0 = none); reset by the host before each launch
__device__ unsigned g_eng_err;

__device__ __forceinline__ bool eng_wait(uint64_t* bar, uint32_t parity, unsigned long long limit_ns,
                                         unsigned where) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255) == 0) {
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      if (*(volatile unsigned*)&g_eng_err) return false;
      if (now - t0 > limit_ns) {
        atomicCAS(&g_eng_err, 0u, where);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------ tensor cores

constexpr int kTcRows = 128;                       // rows per block (MMA M)
constexpr int kTcKTile = 64;                       // K per tile: one 128-byte swizzle row
constexpr int kTcN = 16;                           // MMA N: 8 lanes x (high, low) parts
constexpr int kTcMaxStages = 8;                    // ring of W tiles (fewer when K is large)
constexpr int kTcTileBytes = kTcRows * kTcKTile * 2;  // 16 KiB
constexpr int kTcBTileBytes = kTcN * kTcKTile * 2;    // 2 KiB of activations per K tile
constexpr int kTcThreads = 256;  // warp 0: TMA, warp 1: MMA, warps 4-7: accumulator read-back
constexpr int kTcMaxK = 4096;
constexpr int kTcAccs = 8;       // N = 16 accumulators per buffer: MMA j of tile kt -> (kt & 1) * 4 + j
constexpr int kTcTmemCols = 2 * kTcAccs * kTcN;  // two buffers

constexpr uint32_t kTcIdesc = idesc_bf16(kTcRows, kTcN);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t acc) {
  umma_f16(tmem_d, adesc, bdesc, kTcIdesc, acc);
}

__global__ void __launch_bounds__(kTcThreads, 1)
    tc_matvec_kernel(const __grid_constant__ CUtensorMap wmap, const float* __restrict__ X, int nb, int K,
                     int rows, float* __restrict__ Y, int kTcStages, unsigned long long limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base (the swizzle pattern is taken from address bits)
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int nkt = K / kTcKTile, nblk = rows / kTcRows;
  uint8_t* ring = smem;                                   // kTcStages W tiles
  uint8_t* bsm = ring + kTcStages * kTcTileBytes;         // nkt activation tiles
  uint64_t* full = reinterpret_cast<uint64_t*>(bsm + nkt * kTcBTileBytes);
  uint64_t* empty = full + kTcStages;
  uint64_t* accf = empty + kTcStages;   // accumulator b written (tcgen05.commit)
  uint64_t* acce = accf + 2;            // accumulator b read back (4 warps)
  uint64_t* done = acce + 2;            // every MMA this CTA issued has completed
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&accf[a], 1); mbar_init(&acce[a], 4); }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {  // one full warp allocates the accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // activations as the B operand: row n < 8 is lane n's high part, row 8 + n its low part
  for (int e = threadIdx.x; e < 8 * K; e += kTcThreads) {
    const int n = e / K, k = e % K;
    uint16_t hi = 0, lo = 0;
    if (n < nb) split_bf16(X[(size_t)n * K + k], hi, lo);
    const int kt = k / kTcKTile, kk = k % kTcKTile, c = kk >> 3;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const int row = n + 8 * part;
      const uint32_t off = (uint32_t)(kt * kTcBTileBytes + (row >> 3) * 1024 + (row & 7) * 128 +
                                      ((c ^ (row & 7)) << 4) + (kk & 7) * 2);
      *reinterpret_cast<uint16_t*>(bsm + off) = part ? lo : hi;
    }
  }
  fence_proxy_async_smem();  // the tensor cores read B through the async proxy
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {  // W tiles through the ring
      const uint64_t pol = l2_evict_first_policy();
      uint32_t it = 0;
      bool ok = true;
      for (int blk = blockIdx.x; blk < nblk && ok; blk += gridDim.x)
        for (int kt = 0; kt < nkt && ok; ++kt, ++it) {
          const uint32_t s = it % kTcStages, use = it / kTcStages;
          if (!(ok = eng_wait(&empty[s], (use & 1) ^ 1, limit_ns, 1))) break;
          mbar_arrive_expect_tx(&full[s], kTcTileBytes);
          tma_load_2d(ring + s * kTcTileBytes, &wmap, kt * kTcKTile, blk * kTcRows, &full[s], pol);
        }
      // every copy issued must land before the CTA exits
      const uint32_t first = it > (uint32_t)kTcStages ? it - kTcStages : 0;
      for (uint32_t q = first; q < it; ++q)
        if (!eng_wait(&full[q % kTcStages], (q / kTcStages) & 1, limit_ns, 2)) break;
    }
  } else if (warp == 1) {
    if (lane == 0) {  // the MMA issuer
      uint32_t it = 0;
      int i = 0;
      bool ok = true;
      for (int blk = blockIdx.x; blk < nblk && ok; blk += gridDim.x, ++i) {
        const int a = i & 1, use = i >> 1;
        if (!(ok = eng_wait(&acce[a], (use & 1) ^ 1, limit_ns, 3))) break;
        tc_fence_after();
        for (int kt = 0; kt < nkt; ++kt, ++it) {
          const uint32_t s = it % kTcStages, su = it / kTcStages;
          if (!(ok = eng_wait(&full[s], su & 1, limit_ns, 4))) break;
          tc_fence_after();
          const uint32_t abase = smem_u32(ring + s * kTcTileBytes);
          const uint32_t bbase = smem_u32(bsm + kt * kTcBTileBytes);
#pragma unroll
          for (int j = 0; j < kTcKTile / 16; ++j)
            umma_bf16(tmem + (uint32_t)((a * kTcAccs + (kt & 1) * 4 + j) * kTcN), sw128_desc(abase + j * 32),
                      sw128_desc(bbase + j * 32), kt >= 2 ? 1u : 0u);
          umma_commit(&empty[s]);  // the tile's slot is free once these MMAs have read it
        }
        if (ok) umma_commit(&accf[a]);
      }
      // the CTA must not release tensor memory under MMAs still in flight
      umma_commit(done);
      eng_wait(done, 0, limit_ns, 6);
    }
  } else if (warp >= 4) {  // accumulator read-back: warp 4 + q owns rows 32q .. 32q + 31
    const int q = warp - 4;
    int i = 0;
    for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x, ++i) {
      const int a = i & 1, use = i >> 1;
      if (!eng_wait(&accf[a], use & 1, limit_ns, 5)) break;
      tc_fence_after();
      // the accumulators the block wrote (tiles 0 and 1 start them), two per load
      const int na = nkt >= 2 ? kTcAccs : kTcAccs / 2;
      float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * kTcAccs * kTcN);
      for (int c = 0; c < na; c += 2) {
        uint32_t r[32];
        tmem_ld32(taddr + (uint32_t)(c * kTcN), r);
        tmem_ld_wait();
#pragma unroll
        for (int b = 0; b < 8; ++b)
          y[b] += (__uint_as_float(r[b]) + __uint_as_float(r[8 + b])) +
                  (__uint_as_float(r[16 + b]) + __uint_as_float(r[24 + b]));
      }
      const int row = blk * kTcRows + q * 32 + lane;
#pragma unroll
      for (int b = 0; b < 8; ++b)
        if (b < nb) Y[(size_t)b * rows + row] = y[b];
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[a]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols) : "memory");
}

// ------------------------------------------------------------------ CUDA cores

constexpr int kCcThreads = 288;  // warp 0 lane 0: bulk copies; warps 1-8: dot products
constexpr int kCcPages = 10;     // ring pages (>= 8 consumer warps)

template <int NBT>
__global__ void __launch_bounds__(kCcThreads, 1)
    cc_matvec_kernel(const uint16_t* __restrict__ W, const float* __restrict__ X, int nb, int K, int rows,
                     float* __restrict__ Y, unsigned long long limit_ns) {
  constexpr int RT = 4;  // rows per page (K = 2048)
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  float* act = reinterpret_cast<float*>(ring + kCcPages * kPageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(act + NBT * K);
  uint64_t* empty = full + 2 * kCcPages;
  const int npg = rows / RT;
  const int p0 = (int)((long long)npg * blockIdx.x / gridDim.x), p1 = (int)((long long)npg * (blockIdx.x + 1) / gridDim.x);
  const int n = p1 - p0, nch = K >> 3;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * kCcPages; ++i) mbar_init(&full[i], 1);
    for (int i = 0; i < kCcPages; ++i) mbar_init(&empty[i], kConsumerWarps);
    fence_barrier_init();
  }
  // activations in the split layout mv_core reads (elements 8c..8c+3, then 8c+4..8c+7)
  float4* lo = reinterpret_cast<float4*>(act);
  float4* hi = lo + NBT * nch;
  for (int e = threadIdx.x; e < NBT * nch; e += kCcThreads) {
    const int b = e / nch, c = e % nch;
    float4 l = make_float4(0.f, 0.f, 0.f, 0.f), h = l;
    if (b < nb) {
      l = *reinterpret_cast<const float4*>(X + (size_t)b * K + c * 8);
      h = *reinterpret_cast<const float4*>(X + (size_t)b * K + c * 8 + 4);
    }
    lo[b * nch + c] = l;
    hi[b * nch + c] = h;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t NP = kCcPages;
  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      RingPos rp;
      rp.init(0, NP);
      int k = 0;
      for (; k < n; ++k, rp.advance(1, NP)) {
        if (!eng_wait(&empty[rp.slot], rp.sphase ^ 1u, limit_ns, 11)) break;
        const uint32_t bytes = (uint32_t)RT * K * 2;
        mbar_arrive_expect_tx(&full[rp.fidx], bytes);
        bulk_g2s(ring + (size_t)rp.slot * kPageBytes, W + (size_t)(p0 + k) * RT * K, bytes, &full[rp.fidx], pol);
      }
      const int first = k > (int)NP ? k - (int)NP : 0;
      for (int qq = first; qq < k; ++qq)
        if (!eng_wait(&full[qq % (2 * NP)], (qq / (2 * NP)) & 1, limit_ns, 12)) break;
    }
  } else {
    const int cw = warp - 1;
    const uint32_t alo = smem_u32(act), ahi = alo + (uint32_t)(NBT * nch) * 16u;
    RingPos rp;
    rp.init(cw, NP);
    for (int k = cw; k < n; k += kConsumerWarps, rp.advance(kConsumerWarps, NP)) {
      if (!__all_sync(0xFFFFFFFFu, eng_wait(&full[rp.fidx], rp.fphase, limit_ns, 13))) break;
      float2 acc[RT][NBT];
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int b = 0; b < NBT; ++b) acc[r][b] = make_float2(0.f, 0.f);
      mv_core<RT, NBT>(smem_u32(ring + (size_t)rp.slot * kPageBytes), alo, ahi, nch, lane, acc);
      __syncwarp();
      if (lane == 0) mbar_arrive_cnt(&empty[rp.slot], kConsumerWarps);
      constexpr int NV = RT * NBT;
      float v[NV];
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int b = 0; b < NBT; ++b) v[r * NBT + b] = acc[r][b].x + acc[r][b].y;
      warp_rs<NV, NV, 1, 16>(v, lane);
      constexpr int NL = rs_left(NV, 1);
      const int vbase = rs_base(NV, 1, lane);
      if ((lane & rs_dup_mask(NV, 1)) == 0) {
#pragma unroll
        for (int m = 0; m < NL; ++m) {
          const int idx = vbase + m, r = idx / NBT, b = idx % NBT;
          if (b < nb) Y[(size_t)b * rows + (size_t)(p0 + k) * RT + r] = v[m];
        }
      }
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------ host side

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_eng_mutex;
EncodeTiled g_encode = nullptr;
int g_eng_ready[64];

mk_status eng_setup(int dev) {
  std::lock_guard<std::mutex> lock(g_eng_mutex);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess || !fn ||
        q != cudaDriverEntryPointSuccess)
      return MK_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiled>(fn);
  }
  if (dev < 0 || dev >= 64) return MK_ERR_UNSUPPORTED;
  if (!g_eng_ready[dev]) {
    const int tc_smem = 227 * 1024;
    if (cudaFuncSetAttribute(tc_matvec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc_smem) != cudaSuccess)
      return MK_ERR_CUDA;
    const int cc_smem = kCcPages * kPageBytes + 8 * 2048 * 4 + 8 * 3 * kCcPages;
    const void* ks[4] = {(const void*)cc_matvec_kernel<1>, (const void*)cc_matvec_kernel<2>,
                         (const void*)cc_matvec_kernel<4>, (const void*)cc_matvec_kernel<8>};
    for (auto k : ks)
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, cc_smem) != cudaSuccess)
        return MK_ERR_CUDA;
    g_eng_ready[dev] = 1;
  }
  return MK_OK;
}

}  // namespace

extern "C" mk_status mk_matvec_engine(int32_t engine, const void* W, int32_t rows, int32_t K, const float* X,
                                      int32_t nb, float* Y, int32_t n_sm, int32_t wait_limit_ms, void* stream) {
  if (!W || !X || !Y || nb < 1 || rows < 1 || K < 1) return MK_ERR_INVALID_ARG;
  if (((uintptr_t)W & 15u) || ((uintptr_t)X & 15u)) return MK_ERR_INVALID_ARG;
  if (nb > 8) return MK_ERR_UNSUPPORTED;
  if (engine == 0) {
    if (K != 2048 || rows % 4) return MK_ERR_UNSUPPORTED;
  } else if (engine == 1) {
    if (K % kTcKTile || K > kTcMaxK || rows % kTcRows) return MK_ERR_UNSUPPORTED;
  } else {
    return MK_ERR_INVALID_ARG;
  }
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MK_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MK_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MK_ERR_CUDA;
  if (major != 10) return MK_ERR_UNSUPPORTED;
  mk_status s = eng_setup(dev);
  if (s != MK_OK) return s;
  const int grid_cap = n_sm > 0 && n_sm < sms ? n_sm : sms;
  const unsigned long long limit = (unsigned long long)(wait_limit_ms > 0 ? wait_limit_ms : 1000) * 1000000ull;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaPeekAtLastError() != cudaSuccess) return MK_ERR_CUDA;  // not this call's error to clear
  const unsigned zero = 0;
  if (cudaMemcpyToSymbolAsync(g_eng_err, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return MK_ERR_CUDA;
  if (engine == 1) {
    CUtensorMap map;
    std::memset(&map, 0, sizeof map);
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kTcKTile, (cuuint32_t)kTcRows};
    const cuuint32_t estr[2] = {1, 1};
    if (g_encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MK_ERR_INVALID_ARG;
    const int nblk = rows / kTcRows;
    const int grid = nblk < grid_cap ? nblk : grid_cap;
    const int fixed = 1024 + (K / kTcKTile) * kTcBTileBytes + 256;  // alignment, activations, barriers
    int stages = (227 * 1024 - fixed) / kTcTileBytes;
    if (stages > kTcMaxStages) stages = kTcMaxStages;
    if (stages < 2) return MK_ERR_UNSUPPORTED;
    const int smem = fixed + stages * kTcTileBytes;
    tc_matvec_kernel<<<grid, kTcThreads, smem, st>>>(map, X, nb, K, rows, Y, stages, limit);
  } else {
    const int npg = rows / 4;
    const int grid = npg < grid_cap ? npg : grid_cap;
    const int smem = kCcPages * kPageBytes + 8 * 2048 * 4 + 8 * 3 * kCcPages;
    const int nbt = lanes_template(nb);
    switch (nbt) {
      case 1: cc_matvec_kernel<1><<<grid, kCcThreads, smem, st>>>((const uint16_t*)W, X, nb, K, rows, Y, limit); break;
      case 2: cc_matvec_kernel<2><<<grid, kCcThreads, smem, st>>>((const uint16_t*)W, X, nb, K, rows, Y, limit); break;
      case 4: cc_matvec_kernel<4><<<grid, kCcThreads, smem, st>>>((const uint16_t*)W, X, nb, K, rows, Y, limit); break;
      default: cc_matvec_kernel<8><<<grid, kCcThreads, smem, st>>>((const uint16_t*)W, X, nb, K, rows, Y, limit); break;
    }
  }
  return cudaGetLastError() == cudaSuccess ? MK_OK : MK_ERR_CUDA;
}

extern "C" mk_status mk_matvec_engine_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MK_ERR_CUDA;
  unsigned e = 0;
  if (cudaMemcpyFromSymbol(&e, g_eng_err, sizeof e) != cudaSuccess) return MK_ERR_CUDA;
  return e ? MK_ERR_TIMEOUT : MK_OK;
}
