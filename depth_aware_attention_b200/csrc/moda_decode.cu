// moda_decode.cu -- single-token MoDA decode for B200 (sm_100a).
//
// The operator (hyper.ai summary of arXiv 2603.15619, section "Mixture-of-Depths
// Attention (MoDA)": one jointly normalised softmax over the causal sequence keys and the
// query token's own depth keys), evaluated for ONE query token per sequence: the newest
// token, whose keys/values are the last entry of a cache of S sequence keys.  Its row sees
// every cached key (the causal row of position S-1) and its own L depth keys.  Decoding
// is not on the pages; this is the forward's last row, read as an inference step.
//
// Decode reads each cached K/V byte once and does 4*G FLOPs per K/V element pair: it is
// bound by HBM, so the arithmetic runs on CUDA cores and the work is split over the
// sequence to occupy every SM:
//   1. moda_decode_split_kernel: CTA (bg, split) takes the G query heads of KV group bg
//      over a contiguous range of 128-key blocks (split 0 also the token's depth
//      block(s)).  Warp 4 streams each block's K and V tiles through a TMA ring; warps 0-3
//      compute, one thread per key for the logits (q from shared memory, bf16 x bf16
//      products accumulated in fp32) and one thread per head-dimension column for the
//      P.V sums.  Each head keeps a running max m, normaliser l and fp32 accumulator,
//      written to the workspace at the end.
//   2. moda_decode_combine_kernel: per (bg, head), out = sum_s 2^(m_s - M) acc_s /
//      sum_s 2^(m_s - M) l_s with M = max_s m_s, and lse = (M + log2(den)) * ln 2.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "moda_internal.h"
#include "sm100.cuh"

namespace moda {

namespace {

constexpr int kDecKeys = 128;      // keys per block
constexpr int kDecStages = 3;      // K+V ring stages
constexpr int kDecCompute = 256;   // compute threads (warps 0-7)
constexpr int kDecThreads = kDecCompute + 32;  // and warp 8, the TMA producer
constexpr int kDecMaxG = 16;
constexpr float kLog2eDec = 1.4426950408889634f;
constexpr float kLn2Dec = 0.6931471805599453f;

template <int D>
struct DecCfg {
  static constexpr int kRegions = D / 64;
  static constexpr int kTile = kRegions * 16384;      // 128 keys x D bf16, 128B-swizzled
  static constexpr int kStage = 2 * kTile;            // K then V
  static constexpr int kOffQ = kDecStages * kStage;   // [G][D] bf16, row-major
  static constexpr int kOffP = kOffQ + kDecMaxG * D * 2;  // [8 warps][G][16 keys] fp32
  static constexpr int kOffBar = kOffP + 8 * kDecMaxG * 16 * 4;
  static constexpr int kSmemBytes = 1024 + kOffBar + 128;
  static constexpr int kPairs = D / 64;  // column pairs per thread in the P.V phase
  // the warps' states, [8][G][D] accumulators and [8][G][2] (m, l), reuse the ring after
  // the last block
  static_assert(8 * kDecMaxG * (D + 2) * 4 <= kDecStages * kStage, "ring too small");
};

struct DecArgs {
  const __nv_bfloat16* q;  // [B][Hq][D]
  __nv_bfloat16* out;      // [B][Hq][D]
  float* lse;              // [B][Hq]
  float* ws_acc;           // [BG][nsplit][G][D]
  float* ws_ml;            // [BG][nsplit][G][2]: m (log2 units), l
  int B, Hq, Hkv, S, L, G, nsplit, bps;  // bps: sequence blocks per split
  // Groups above kDecMaxG heads run the split kernel once per chunk of at most kDecMaxG
  // heads (each launch reads the K/V cache again): G is the chunk's head count, head0 its
  // first head, Gfull the group size, which the workspace and the combine kernel index by.
  int head0, Gfull;
  float scale_log2;
};

struct DecBars {
  uint64_t full[kDecStages], empty[kDecStages];
  int abort;
};

// Byte offset of 16-byte chunk c of row r in a 128B-swizzled 64-column region.
__device__ __forceinline__ uint32_t dec_sw(int r, int c) {
  return uint32_t(r) * 128u + ((uint32_t(c) ^ (uint32_t(r) & 7u)) << 4);
}

__device__ __forceinline__ uint32_t lds_b32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// GM: group size rounded up to a power of two (loop bound); kExact: G == GM.
// Warp 8 streams each block's K and V tiles through the TMA ring.  Compute warp w owns keys
// [16w, 16w + 16) of every block and keeps its own online-softmax state (running max m,
// normaliser l, fp32 accumulator) for the G heads over the whole split, so the eight
// warps never wait for each other within a block:
//   logits: two lanes per key, each over half the head dimension (q from shared memory,
//           bf16 x bf16 products accumulated in fp32), finished with one shuffle;
//   P.V:    each lane owns column pairs (2 lane, 2 lane + 64 for D = 128) and reads V as
//           packed bf16 pairs, with packed f32x2 FMAs, over the warp's 16 keys.
// After the last block the eight states are merged exactly (each rescaled to the largest
// max) and written to the workspace.
template <int D, int GM, bool kExact>
__global__ void __launch_bounds__(kDecThreads, 1)
    moda_decode_split_kernel(const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV,
                             const __grid_constant__ CUtensorMap tmKD,
                             const __grid_constant__ CUtensorMap tmVD, const DecArgs a) {
  using Cfg = DecCfg<D>;
  extern __shared__ uint8_t dec_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dec_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s0 = smem_u32(smem);
  DecBars* bars = reinterpret_cast<DecBars*>(smem + Cfg::kOffBar);
  volatile int* abort_flag = &bars->abort;
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };

  const int bg = blockIdx.x / a.nsplit;
  const int split = blockIdx.x - bg * a.nsplit;
  const int G = kExact ? GM : a.G;
  const int nseq = (a.S + kDecKeys - 1) / kDecKeys;
  const int sb0 = split * a.bps;
  const int sb1 = min(nseq, sb0 + a.bps);
  const int ndep = (split == 0 && a.L > 0) ? (a.L + kDecKeys - 1) / kDecKeys : 0;
  const int nblk = ndep + (sb1 - sb0);  // depth blocks first, then sequence blocks
  const int warp = threadIdx.x >> 5;
  // the combine grid may be scheduled now: it waits for this grid's completion itself
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(bar(bars->full[s]), 1);
      mbar_init(bar(bars->empty[s]), kDecCompute);
    }
    bars->abort = 0;
    fence_barrier_init();
  }
  // the G query rows of this chunk (bf16) into shared memory
  const int b = bg / a.Hkv, g = bg - (bg / a.Hkv) * a.Hkv;
  for (int i = threadIdx.x; i < G * D / 8; i += kDecThreads) {
    const int h = i / (D / 8), c = i - h * (D / 8);
    const uint4 w = ldg_nc_v4(a.q + ((size_t(b) * a.Hq + g * a.Gfull + a.head0 + h) * D + c * 8));
    sts128(s0 + Cfg::kOffQ + uint32_t((h * D + c * 8) * 2), w);
  }
  __syncthreads();

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int i = 0; i < nblk; ++i) {
        const int s = i % kDecStages;
        if (i >= kDecStages &&
            !mbar_wait(bar(bars->empty[s]), ((i / kDecStages) - 1) & 1, abort_flag))
          break;
        mbar_expect_tx(bar(bars->full[s]), Cfg::kStage);
        const bool dep = i < ndep;
        const int row0 = dep ? i * kDecKeys : (sb0 + i - ndep) * kDecKeys;
        const uint32_t st = s0 + uint32_t(s) * Cfg::kStage;
        for (int rg = 0; rg < Cfg::kRegions; ++rg) {
          tma_load_3d(st + rg * 16384, dep ? &tmKD : &tmK, bar(bars->full[s]), rg * 64, row0,
                      bg);
          tma_load_3d(st + Cfg::kTile + rg * 16384, dep ? &tmVD : &tmV, bar(bars->full[s]),
                      rg * 64, row0, bg);
        }
      }
    }
    __syncwarp();
    return;  // the producer warp takes no part in the compute warps' barriers
  }

  // ------------------------------------------------------------ compute warps 0-7
  const int lane = threadIdx.x & 31;
  const int kl = lane >> 1, part = lane & 1;  // the lane's key among the warp's 16, half of D
  const int key = 16 * warp + kl;             // key of the block
  constexpr int kChunks = D / 16;             // 16-byte chunks of a lane's half row
  constexpr int NP = Cfg::kPairs;
  const uint32_t pw = s0 + Cfg::kOffP + uint32_t(warp * kDecMaxG * 16 * 4);  // [G][16] fp32
  float* Pw = reinterpret_cast<float*>(smem + Cfg::kOffP) + warp * kDecMaxG * 16;
  float m[GM], l[GM];
  float2 acc[GM][NP];
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int j = 0; j < NP; ++j) acc[h][j] = make_float2(0.f, 0.f);
  }
  for (int i = 0; i < nblk; ++i) {
    const int s = i % kDecStages;
    mbar_wait(bar(bars->full[s]), (i / kDecStages) & 1, abort_flag);
    const uint32_t kst = s0 + uint32_t(s) * Cfg::kStage;
    const uint32_t vst = kst + Cfg::kTile;
    const bool dep = i < ndep;
    const int kabs = (dep ? i : sb0 + i - ndep) * kDecKeys + key;
    const bool kvalid = kabs < (dep ? a.L : a.S);
    // logits of this key for the G heads (this lane's half of the dot products)
    float y[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) y[h] = 0.f;
#pragma unroll
    for (int cc = 0; cc < kChunks; ++cc) {
      const int ch = part * kChunks + cc;  // 16-byte chunk of the row
      const uint4 kw = lds128(kst + (ch / 8) * 16384 + dec_sw(key, ch % 8));
#pragma unroll
      for (int h = 0; h < GM; ++h)
        if (h < G)
          y[h] = dot8_bf16(lds128(s0 + Cfg::kOffQ + uint32_t((h * D + ch * 8) * 2)), kw, y[h]);
    }
    // the warp's online-softmax step over its 16 keys
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      if (h < G) {
        y[h] += __shfl_xor_sync(0xffffffffu, y[h], 1);
        const float yv = kvalid ? y[h] * a.scale_log2 : -INFINITY;
        float bmax = yv;
#pragma unroll
        for (int o = 16; o > 1; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
        const float m_new = fmaxf(m[h], bmax);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = ex2(m[h] - m_use);
        const float p = ex2(yv - m_use);
        if (part == 0) Pw[h * 16 + kl] = p;
        float sum = part == 0 ? p : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        l[h] = l[h] * alpha + sum;
        m[h] = m_new;
#pragma unroll
        for (int j = 0; j < NP; ++j) acc[h][j] = fmul2(acc[h][j], make_float2(alpha, alpha));
      }
    }
    __syncwarp();  // P of the warp's keys written
    // P.V over the warp's 16 keys: column pairs 2 lane + 64 j
#pragma unroll 2
    for (int k4 = 0; k4 < 16; k4 += 4) {
      float2 vv[4][NP];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int j = 0; j < NP; ++j) {
          const int col = 2 * lane + 64 * j;
          const uint32_t w = lds_b32(vst + uint32_t((col / 64) * 16384 + (col % 8) * 2) +
                                     dec_sw(16 * warp + k4 + u, (col % 64) / 8));
          vv[u][j] = make_float2(bf16lo(w), bf16hi(w));
        }
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        if (h < G) {
          const uint4 pq = lds128(pw + uint32_t((h * 16 + k4) * 4));
          const float pk[4] = {__uint_as_float(pq.x), __uint_as_float(pq.y),
                               __uint_as_float(pq.z), __uint_as_float(pq.w)};
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int j = 0; j < NP; ++j)
              acc[h][j] = ffma2(make_float2(pk[u], pk[u]), vv[u][j], acc[h][j]);
        }
      }
    }
    __syncwarp();  // the warp's P is rewritten by the next block
    mbar_arrive(bar(bars->empty[s]));
  }

  // merge the eight warps' states in the ring's memory: free once every warp has finished
  // reading its last block (every block's loads were waited for)
  named_bar_sync(1, kDecCompute);
  float* wacc = reinterpret_cast<float*>(smem);          // [8][G][D]
  float* wml = wacc + 8 * kDecMaxG * D;                   // [8][G][2]
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    if (h < G) {
#pragma unroll
      for (int j = 0; j < NP; ++j)
        *reinterpret_cast<float2*>(wacc + (warp * kDecMaxG + h) * D + 2 * lane + 64 * j) =
            acc[h][j];
      if (lane == 0) {
        wml[(warp * kDecMaxG + h) * 2] = m[h];
        wml[(warp * kDecMaxG + h) * 2 + 1] = l[h];
      }
    }
  }
  named_bar_sync(1, kDecCompute);
  const size_t base = (size_t(bg) * a.nsplit + split) * a.Gfull + a.head0;
  for (int e = threadIdx.x; e < G * (D / 2); e += kDecCompute) {
    const int h = e / (D / 2), col = 2 * (e - h * (D / 2));
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) M = fmaxf(M, wml[(w * kDecMaxG + h) * 2]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float2 v = make_float2(0.f, 0.f);
    float lsum = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const float f = ex2(wml[(w * kDecMaxG + h) * 2] - Mu);
      const float2 x = *reinterpret_cast<const float2*>(wacc + (w * kDecMaxG + h) * D + col);
      v.x = fmaf(f, x.x, v.x);
      v.y = fmaf(f, x.y, v.y);
      lsum = fmaf(f, wml[(w * kDecMaxG + h) * 2 + 1], lsum);
    }
    *reinterpret_cast<float2*>(a.ws_acc + (base + h) * D + col) = v;
    if (col == 0) {
      a.ws_ml[(base + h) * 2] = M;
      a.ws_ml[(base + h) * 2 + 1] = lsum;
    }
  }
}

constexpr int kDecMaxSplit = 256;

// One CTA per (bg, head), thread = head-dimension column.  The splits' (m, l) are staged
// in shared memory and their weights computed once; the accumulator loads of all splits
// are independent, so several are kept in flight.
template <int D>
__global__ void __launch_bounds__(D) moda_decode_combine_kernel(const DecArgs a) {
  __shared__ float wgt[kDecMaxSplit], lsp[kDecMaxSplit];
  __shared__ float mmax;
  const int bg = blockIdx.x / a.Gfull, h = blockIdx.x - (blockIdx.x / a.Gfull) * a.Gfull;
  const int d = threadIdx.x;
  const size_t base = size_t(bg) * a.nsplit * a.Gfull;
  const int ns = a.nsplit;
  // the split grid's partials: wait for its completion (a no-op for an ordinary launch)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int s = d; s < ns; s += D) {
    const size_t r = base + size_t(s) * a.Gfull + h;
    wgt[s] = a.ws_ml[r * 2];
    lsp[s] = a.ws_ml[r * 2 + 1];
  }
  __syncthreads();
  if (d < 32) {
    float M = -INFINITY;
    for (int s = d; s < ns; s += 32) M = fmaxf(M, wgt[s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (d == 0) mmax = (M == -INFINITY) ? 0.f : M;
  }
  __syncthreads();
  const float Mu = mmax;
  for (int s = d; s < ns; s += D) wgt[s] = ex2(wgt[s] - Mu);
  __syncthreads();
  float den = 0.f, n0 = 0.f, n1 = 0.f, n2 = 0.f, n3 = 0.f;
  const float* accp = a.ws_acc + base * D + size_t(h) * D + d;  // split s at + s * G * D
  const size_t stride = size_t(a.Gfull) * D;
  int s = 0;
  for (; s + 16 <= ns; s += 16) {  // sixteen independent loads in flight
    float x[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) x[u] = accp[size_t(s + u) * stride];
#pragma unroll
    for (int u = 0; u < 16; u += 4) {
      n0 = fmaf(wgt[s + u], x[u], n0);
      n1 = fmaf(wgt[s + u + 1], x[u + 1], n1);
      n2 = fmaf(wgt[s + u + 2], x[u + 2], n2);
      n3 = fmaf(wgt[s + u + 3], x[u + 3], n3);
    }
  }
  for (; s + 4 <= ns; s += 4) {
    const float x0 = accp[size_t(s) * stride], x1 = accp[size_t(s + 1) * stride];
    const float x2 = accp[size_t(s + 2) * stride], x3 = accp[size_t(s + 3) * stride];
    n0 = fmaf(wgt[s], x0, n0);
    n1 = fmaf(wgt[s + 1], x1, n1);
    n2 = fmaf(wgt[s + 2], x2, n2);
    n3 = fmaf(wgt[s + 3], x3, n3);
  }
  for (; s < ns; ++s) n0 = fmaf(wgt[s], accp[size_t(s) * stride], n0);
  for (int t = 0; t < ns; ++t) den = fmaf(wgt[t], lsp[t], den);
  const int b = bg / a.Hkv, g = bg - (bg / a.Hkv) * a.Hkv;
  const size_t row = size_t(b) * a.Hq + g * a.Gfull + h;
  a.out[row * D + d] = __float2bfloat16_rn(((n0 + n1) + (n2 + n3)) / den);
  if (d == 0) a.lse[row] = (Mu + __log2f(den)) * kLn2Dec;
}

bool make_map_dec(EncodeTiledFn encode, CUtensorMap* map, const void* base, cuuint64_t D,
                  cuuint64_t rows, cuuint64_t BG) {
  const cuuint64_t dims[3] = {D, rows, BG};
  const cuuint64_t str[2] = {D * 2, rows * D * 2};
  const cuuint32_t box[3] = {64, kDecKeys, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, str,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_decode_d(const Problem& p, const DecodeSplit& sp, const void* q,
                            const void* k, const void* v, const void* kd, const void* vd,
                            void* out, float* lse, void* workspace, EncodeTiledFn encode,
                            cudaStream_t stream, const char** why) {
  using Cfg = DecCfg<D>;
  const cuuint64_t BG = cuuint64_t(p.B) * p.Hkv;
  CUtensorMap mK, mV, mKD, mVD;
  if (!make_map_dec(encode, &mK, k, D, cuuint64_t(p.T), BG) ||
      !make_map_dec(encode, &mV, v, D, cuuint64_t(p.T), BG)) {
    *why = "cuTensorMapEncodeTiled failed for the K/V cache";
    return cudaErrorInvalidValue;
  }
  if (p.L > 0) {
    if (!make_map_dec(encode, &mKD, kd, D, cuuint64_t(p.L), BG) ||
        !make_map_dec(encode, &mVD, vd, D, cuuint64_t(p.L), BG)) {
      *why = "cuTensorMapEncodeTiled failed for kd/vd";
      return cudaErrorInvalidValue;
    }
  } else {
    mKD = mK;  // never loaded when L == 0
    mVD = mV;
  }
  DecArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.ws_acc = static_cast<float*>(workspace);
  a.ws_ml = a.ws_acc + size_t(BG) * sp.nsplit * p.G * D;
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.S = p.T;
  a.L = p.L;
  a.G = p.G;
  a.head0 = 0;
  a.Gfull = p.G;
  a.nsplit = sp.nsplit;
  a.bps = sp.blocks_per_split;
  a.scale_log2 = p.scale * kLog2eDec;
  auto run = [&](auto kern) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           Cfg::kSmemBytes);
    if (err != cudaSuccess) return err;
    kern<<<unsigned(BG) * sp.nsplit, kDecThreads, Cfg::kSmemBytes, stream>>>(mK, mV, mKD,
                                                                            mVD, a);
    return cudaGetLastError();
  };
  cudaError_t e = cudaSuccess;
  for (a.head0 = 0; a.head0 < p.G && e == cudaSuccess; a.head0 += kDecMaxG) {
    a.G = min(kDecMaxG, p.G - a.head0);  // heads of this chunk
    switch (a.G) {
      case 1: e = run(moda_decode_split_kernel<D, 1, true>); break;
      case 2: e = run(moda_decode_split_kernel<D, 2, true>); break;
      case 3: e = run(moda_decode_split_kernel<D, 4, false>); break;
      case 4: e = run(moda_decode_split_kernel<D, 4, true>); break;
      case 8: e = run(moda_decode_split_kernel<D, 8, true>); break;
      case 16: e = run(moda_decode_split_kernel<D, 16, true>); break;
      default:
        e = a.G < 8 ? run(moda_decode_split_kernel<D, 8, false>)
                    : run(moda_decode_split_kernel<D, 16, false>);
    }
  }
  if (e != cudaSuccess) {
    *why = "decode split kernel launch failed";
    return e;
  }
  {
    // programmatic dependent launch: the combine grid is scheduled while the split grid
    // runs (it triggers at its start) and waits for the split grid's completion and
    // memory in its first instruction, so the launch gap overlaps the split grid's tail
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(BG) * a.Gfull);
    cfg.blockDim = dim3(D);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, moda_decode_combine_kernel<D>, a);
    if (e != cudaSuccess) {
      *why = "decode combine kernel launch failed";
      return e;
    }
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) *why = "decode combine kernel launch failed";
  return e;
}

}  // namespace

DecodeSplit decode_split(const Problem& p) {
  // One CTA (about 206 KB of shared memory) per SM of a B200 (148 SMs).  The split count
  // is chosen so that the CTAs fill whole waves: among splits of up to 8 waves the one with
  // the least idle SM time, each wave beyond the first charged 1% (every CTA refills its
  // load pipeline).  The choice depends on the sizes alone, so the workspace size is a
  // function of the sizes.
  constexpr int kSMs = 148, kMaxWaves = 8;
  DecodeSplit sp;
  const int nseq = (p.T + kDecKeys - 1) / kDecKeys;
  const long long bg = (long long)p.B * p.Hkv;
  int best_ns = 1;
  double best_eff = -1.0;
  long long best_waves = 0;
  const int max_ns = min(nseq, kDecMaxSplit);
  for (int want = 1; want <= max_ns; ++want) {
    const int bps = (nseq + want - 1) / want;
    const int ns = (nseq + bps - 1) / bps;  // no empty split
    const long long ctas = bg * ns;
    const long long waves = (ctas + kSMs - 1) / kSMs;
    if (waves > kMaxWaves && want > 1) break;
    const double eff = double(ctas) / double(waves * kSMs) - 0.01 * double(waves - 1);
    if (eff > best_eff + 1e-9 || (eff > best_eff - 1e-9 && waves < best_waves)) {
      best_eff = eff;
      best_ns = ns;
      best_waves = waves;
    }
  }
  sp.blocks_per_split = (nseq + best_ns - 1) / best_ns;
  sp.nsplit = (nseq + sp.blocks_per_split - 1) / sp.blocks_per_split;
  return sp;
}

size_t decode_workspace_bytes(const Problem& p) {
  const DecodeSplit sp = decode_split(p);
  const size_t n = size_t(p.B) * p.Hkv * sp.nsplit * p.G;
  return n * p.d * 4 + n * 2 * 4 + 256;
}

cudaError_t launch_decode(const Problem& p, const void* q, const void* k, const void* v,
                          const void* kd, const void* vd, void* out, float* lse,
                          void* workspace, EncodeTiledFn encode, cudaStream_t stream,
                          const char** why) {
  const DecodeSplit sp = decode_split(p);
  if (p.d == 128)
    return launch_decode_d<128>(p, sp, q, k, v, kd, vd, out, lse, workspace, encode, stream,
                                why);
  return launch_decode_d<64>(p, sp, q, k, v, kd, vd, out, lse, workspace, encode, stream, why);
}

}  // namespace moda
