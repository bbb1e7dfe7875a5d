// moda_kvwrite.cu -- fused depth-stream write for B200 (sm_100a).
//
// Every sublayer appends its key/value pair to the depth stream that later layers read
// (hyper.ai summary of arXiv 2603.15619, section "Hardware-efficient implementation":
// the depth cache is kept flattened per (batch, KV head) so that token t's entries are
// the contiguous rows [t*L, (t+1)*L), layout [B, Hkv, T, L, d]).  This kernel is the
// projection that produces layer l's pair, K|V = X W^T, with the depth cache as its
// epilogue: each token's K and V rows go straight into slot l of kd / vd, with no
// separate copy of a [B*T, 2*Hkv*d] product.
//
// Tiles of 128 tokens x 256 columns of X W^T on the tensor cores, a persistent CTA per SM
// walking its share of the tiles:
//   warp 4     TMA producer: 64-wide K-slices of the X tile (128 rows) and the W tile
//              (256 rows; both K-major, 128B-swizzled) through a ring of shared-memory
//              stages;
//   warp 5     tcgen05 issuer: four 128x256x16 MMAs per stage into a 256-column TMEM
//              accumulator, the stage released by a commit once they are done;
//   warps 0-3  epilogue: TMEM lane r = the tile's token r; each 32-column chunk lies in
//              one head of K or of V, converted to bf16 and stored as contiguous 16-byte
//              words into the token's slot-l row.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moda_internal.h"
#include "sm100.cuh"

namespace moda {

namespace {

constexpr int kKwRows = 128;    // tokens per tile
constexpr int kKwCols = 256;    // output columns per tile
constexpr int kKwBK = 64;       // K (hidden) elements per stage: 128 bytes per row
constexpr int kKwStages = 4;
constexpr int kKwThreads = 192; // warps 0-3 epilogue, 4 producer, 5 issuer
constexpr int kKwTile = 16384;  // 128 rows x 128 bytes: the x slice; the W slice is two

struct KwArgs {
  __nv_bfloat16 *kd, *vd;
  int M, T, hidden, Hkv, d, L, slot, nk;
  int ntn, ntiles;  // column tiles per row tile; all tiles
};

struct KwBars {
  uint64_t full[kKwStages], empty[kKwStages];
  uint64_t acc_full[2], acc_empty[2];  // TMEM accumulator buffers
  uint32_t tmem_base;
  int abort;
};

constexpr int kKwStage = 3 * kKwTile;  // x slice (128 rows) + W slice (256 rows)
constexpr int kKwOffBar = kKwStages * kKwStage;
constexpr int kKwSmemBytes = 1024 + kKwOffBar + 256;

// Persistent: CTA c takes tiles c, c + gridDim.x, ... (column tiles innermost, so
// consecutive tiles reuse the x rows from L2).  The shared-memory ring runs on across
// tiles, and the TMEM accumulator is double-buffered (2 x 256 columns), so one tile's
// epilogue overlaps the next tile's main loop.
__global__ void __launch_bounds__(kKwThreads, 1)
    moda_kvwrite_kernel(const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmW, const KwArgs a) {
  extern __shared__ uint8_t kw_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(kw_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s0 = smem_u32(smem);
  KwBars* bars = reinterpret_cast<KwBars*>(smem + kKwOffBar);
  volatile int* abort_flag = &bars->abort;
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };
  auto sA = [&](int s) { return s0 + uint32_t(s) * kKwStage; };
  auto sB = [&](int s) { return s0 + uint32_t(s) * kKwStage + kKwTile; };

  const int warp = threadIdx.x >> 5;
  const int nmine = a.ntiles > int(blockIdx.x)
                        ? (a.ntiles - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x)
                        : 0;
  auto tile_of = [&](int j, int& m0, int& n0) {
    const int t = int(blockIdx.x) + j * int(gridDim.x);
    m0 = (t / a.ntn) * kKwRows;
    n0 = (t - (t / a.ntn) * a.ntn) * kKwCols;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKwStages; ++s) {
      mbar_init(bar(bars->full[s]), 1);
      mbar_init(bar(bars->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(bars->acc_full[b]), 1);
      mbar_init(bar(bars->acc_empty[b]), 128);
    }
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(&bars->tmem_base), 2 * kKwCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmW);
      int g = 0;  // k-block counter across tiles
      for (int j = 0; j < nmine; ++j) {
        int m0, n0;
        tile_of(j, m0, n0);
        for (int kb = 0; kb < a.nk; ++kb, ++g) {
          const int s = g % kKwStages;
          if (g >= kKwStages)
            mbar_wait(bar(bars->empty[s]), ((g / kKwStages) - 1) & 1, abort_flag);
          mbar_expect_tx(bar(bars->full[s]), kKwStage);
          tma_load_2d(sA(s), &tmX, bar(bars->full[s]), kb * kKwBK, m0);
          tma_load_2d(sB(s), &tmW, bar(bars->full[s]), kb * kKwBK, n0);
          tma_load_2d(sB(s) + kKwTile, &tmW, bar(bars->full[s]), kb * kKwBK, n0 + 128);
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ tcgen05 issuer
    if (elect_one()) {
      constexpr uint32_t idesc = make_idesc_bf16(kKwRows, kKwCols, 0, 0);
      int g = 0;
      for (int j = 0; j < nmine; ++j) {
        const int ab = j & 1;
        const uint32_t acc = tmem + uint32_t(ab * kKwCols);
        if (j >= 2) mbar_wait(bar(bars->acc_empty[ab]), ((j >> 1) - 1) & 1, abort_flag);
        tc_fence_after();
        for (int kb = 0; kb < a.nk; ++kb, ++g) {
          const int s = g % kKwStages;
          mbar_wait(bar(bars->full[s]), (g / kKwStages) & 1, abort_flag);
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < kKwBK / 16; ++ks)
            mma_ss(acc, make_sdesc_sw128(sA(s) + ks * 32, 16, 1024),
                   make_sdesc_sw128(sB(s) + ks * 32, 16, 1024), idesc,
                   (kb > 0 || ks > 0) ? 1u : 0u);
          tc_commit(bar(bars->empty[s]));
        }
        tc_commit(bar(bars->acc_full[ab]));
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue warps 0-3
    const int r = threadIdx.x;  // TMEM lane = row r of the tile
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const int hd = a.Hkv * a.d;
    for (int j = 0; j < nmine; ++j) {
      const int ab = j & 1;
      int m0, n0;
      tile_of(j, m0, n0);
      mbar_wait(bar(bars->acc_full[ab]), (j >> 1) & 1, abort_flag);
      tc_fence_after();
      const int m = m0 + r;
      const bool valid = m < a.M;
      const int b = valid ? m / a.T : 0, t = valid ? m - (m / a.T) * a.T : 0;
#pragma unroll
      for (int cc = 0; cc < kKwCols / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tmem + uint32_t(ab * kKwCols) + lane_base + cc * 32, o);
        tmem_wait_ld();
        if (valid) {
          const int na = n0 + cc * 32;
          const int part = na / hd;  // 0: K columns, 1: V columns
          __nv_bfloat16* base = part ? a.vd : a.kd;
          const int n = na - part * hd;  // column within K (or V)
          const int g = n / a.d, c = n - g * a.d;
          uint4* dst = reinterpret_cast<uint4*>(
              base + ((((size_t(b) * a.Hkv + g) * a.T + t) * a.L + a.slot) * a.d + c));
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(o[v4 * 8 + e]);
            dst[v4] = pack8(f, 1.f);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(bars->acc_empty[ab]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kKwCols);
  }
}

bool make_map_2d(EncodeTiledFn encode, CUtensorMap* map, const void* base, cuuint64_t inner,
                 cuuint64_t rows) {
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t str[1] = {inner * 2};
  const cuuint32_t box[2] = {kKwBK, 128};
  cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, str,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_kvwrite(const KvWriteProblem& p, const void* x, const void* w, void* kd,
                           void* vd, EncodeTiledFn encode, cudaStream_t stream,
                           const char** why) {
  const int M = p.B * p.T, N = 2 * p.Hkv * p.d;
  CUtensorMap mX, mW;
  if (!make_map_2d(encode, &mX, x, cuuint64_t(p.hidden), cuuint64_t(M)) ||
      !make_map_2d(encode, &mW, w, cuuint64_t(p.hidden), cuuint64_t(N))) {
    *why = "cuTensorMapEncodeTiled failed for x/w";
    return cudaErrorInvalidValue;
  }
  KwArgs a;
  a.kd = static_cast<__nv_bfloat16*>(kd);
  a.vd = static_cast<__nv_bfloat16*>(vd);
  a.M = M;
  a.T = p.T;
  a.hidden = p.hidden;
  a.Hkv = p.Hkv;
  a.d = p.d;
  a.L = p.L;
  a.slot = p.slot;
  a.nk = (p.hidden + kKwBK - 1) / kKwBK;
  a.ntn = N / kKwCols;
  a.ntiles = ((M + kKwRows - 1) / kKwRows) * a.ntn;
  cudaError_t e = cudaFuncSetAttribute(moda_kvwrite_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kKwSmemBytes);
  if (e != cudaSuccess) {
    *why = "cudaFuncSetAttribute(depth-stream write) failed";
    return e;
  }
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int grid = a.ntiles < nsm ? a.ntiles : nsm;  // persistent: one CTA per SM
  moda_kvwrite_kernel<<<grid, kKwThreads, kKwSmemBytes, stream>>>(mX, mW, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) *why = "depth-stream write launch failed";
  return e;
}

}  // namespace moda
