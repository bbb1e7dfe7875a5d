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
constexpr int kDecThreads = 160;   // warps 0-3 compute, warp 4 TMA producer
constexpr int kDecMaxG = 16;
constexpr float kLog2eDec = 1.4426950408889634f;
constexpr float kLn2Dec = 0.6931471805599453f;

template <int D>
struct DecCfg {
  static constexpr int kRegions = D / 64;
  static constexpr int kTile = kRegions * 16384;      // 128 keys x D bf16, 128B-swizzled
  static constexpr int kStage = 2 * kTile;            // K then V
  static constexpr int kOffQ = kDecStages * kStage;   // [G][D] bf16, row-major
  static constexpr int kOffP = kOffQ + kDecMaxG * D * 2;           // [G][128] fp32
  static constexpr int kOffRed = kOffP + kDecMaxG * kDecKeys * 4;  // [2][4][G] fp32
  static constexpr int kOffAcc = kOffRed + 2 * 4 * kDecMaxG * 4;   // [G][D] fp32 (D = 64)
  static constexpr int kOffBar = kOffAcc + (D == 64 ? kDecMaxG * D * 4 : 0);
  static constexpr int kSmemBytes = 1024 + kOffBar + 128;
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

// GM: group size rounded up to a power of two (loop bound); kExact: G == GM.
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
  float* P = reinterpret_cast<float*>(smem + Cfg::kOffP);
  float* red = reinterpret_cast<float*>(smem + Cfg::kOffRed);

  const int bg = blockIdx.x / a.nsplit;
  const int split = blockIdx.x - bg * a.nsplit;
  const int G = kExact ? GM : a.G;
  const int nseq = (a.S + kDecKeys - 1) / kDecKeys;
  const int sb0 = split * a.bps;
  const int sb1 = min(nseq, sb0 + a.bps);
  const int ndep = (split == 0 && a.L > 0) ? (a.L + kDecKeys - 1) / kDecKeys : 0;
  const int nblk = ndep + (sb1 - sb0);  // depth blocks first, then sequence blocks
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(bar(bars->full[s]), 1);
      mbar_init(bar(bars->empty[s]), 128);
    }
    bars->abort = 0;
    fence_barrier_init();
  }
  // the G query rows of this group (bf16) into shared memory
  const int b = bg / a.Hkv, g = bg - (bg / a.Hkv) * a.Hkv;
  for (int i = threadIdx.x; i < G * D / 8; i += kDecThreads) {
    const int h = i / (D / 8), c = i - h * (D / 8);
    const uint4 w = ldg_nc_v4(a.q + ((size_t(b) * a.Hq + g * a.Gfull + a.head0 + h) * D + c * 8));
    sts128(s0 + Cfg::kOffQ + uint32_t((h * D + c * 8) * 2), w);
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int i = 0; i < nblk; ++i) {
        const int s = i % kDecStages;
        if (i >= kDecStages)
          mbar_wait(bar(bars->empty[s]), ((i / kDecStages) - 1) & 1, abort_flag);
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

  // ------------------------------------------------------------ compute warps 0-3
  const int tid = threadIdx.x;              // key of the block (logit phase)
  constexpr int KG = 128 / D;               // key groups in the P.V phase
  const int dcol = tid % D, kg = tid / D;   // head-dimension column, key group
  const int lane = tid & 31;
  float m[GM], l[GM], acc[GM];
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
    acc[h] = 0.f;
  }
  for (int i = 0; i < nblk; ++i) {
    const int s = i % kDecStages;
    mbar_wait(bar(bars->full[s]), (i / kDecStages) & 1, abort_flag);
    const uint32_t kst = s0 + uint32_t(s) * Cfg::kStage;
    const uint32_t vst = kst + Cfg::kTile;
    const bool dep = i < ndep;
    const int kabs = (dep ? i : sb0 + i - ndep) * kDecKeys + tid;
    const bool kvalid = kabs < (dep ? a.L : a.S);
    // logits of this key for the G heads
    float y[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) y[h] = 0.f;
#pragma unroll
    for (int rg = 0; rg < Cfg::kRegions; ++rg) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 kw = lds128(kst + rg * 16384 + dec_sw(tid, c));
#pragma unroll
        for (int h = 0; h < GM; ++h)
          if (h < G)
            y[h] = dot8_bf16(lds128(s0 + Cfg::kOffQ + uint32_t((h * D + rg * 64 + c * 8) * 2)),
                             kw, y[h]);
      }
    }
    // block max per head: warp max, then across the four warps
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      if (h < G) {
        y[h] = kvalid ? y[h] * a.scale_log2 : -INFINITY;
        float v = y[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[warp * kDecMaxG + h] = v;
      }
    }
    named_bar_sync(1, 128);
    float alpha[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      alpha[h] = 1.f;
      if (h < G) {
        const float bmax = fmaxf(fmaxf(red[h], red[kDecMaxG + h]),
                                 fmaxf(red[2 * kDecMaxG + h], red[3 * kDecMaxG + h]));
        const float m_new = fmaxf(m[h], bmax);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[h] = ex2(m[h] - m_use);
        const float p = ex2(y[h] - m_use);
        P[h * kDecKeys + tid] = p;
        float v = p;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[(4 + warp) * kDecMaxG + h] = v;
        m[h] = m_new;
      }
    }
    named_bar_sync(1, 128);
    // P.V: column dcol over this thread's key group
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      if (h < G) {
        const float bsum = (red[4 * kDecMaxG + h] + red[5 * kDecMaxG + h]) +
                           (red[6 * kDecMaxG + h] + red[7 * kDecMaxG + h]);
        l[h] = l[h] * alpha[h] + bsum;
        acc[h] *= alpha[h];
      }
    }
    {
      const int rg = dcol / 64, col = dcol % 64;
      const uint32_t vcol = vst + rg * 16384 + uint32_t(col % 8) * 2;
      const uint32_t pbase = s0 + Cfg::kOffP;
      constexpr int NK = kDecKeys / KG;  // keys of this thread's group
#pragma unroll 2
      for (int k4 = 0; k4 < NK; k4 += 4) {
        const int k = kg * NK + k4;
        float vv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) vv[u] = bf16lo(lds_u16(vcol + dec_sw(k + u, col / 8)));
#pragma unroll
        for (int h = 0; h < GM; ++h) {
          if (h < G) {
            const uint4 pw = lds128(pbase + uint32_t(h * kDecKeys + k) * 4u);
            acc[h] = fmaf(__uint_as_float(pw.x), vv[0], acc[h]);
            acc[h] = fmaf(__uint_as_float(pw.y), vv[1], acc[h]);
            acc[h] = fmaf(__uint_as_float(pw.z), vv[2], acc[h]);
            acc[h] = fmaf(__uint_as_float(pw.w), vv[3], acc[h]);
          }
        }
      }
    }
    named_bar_sync(1, 128);  // P and the reduction slots are rewritten by the next block
    mbar_arrive(bar(bars->empty[s]));
  }

  // partial results of this split
  float* accs = reinterpret_cast<float*>(smem + Cfg::kOffAcc);
  if (KG == 2) {
    if (kg == 1) {
#pragma unroll
      for (int h = 0; h < GM; ++h)
        if (h < G) accs[h * D + dcol] = acc[h];
    }
    named_bar_sync(1, 128);
  }
  if (kg == 0) {
    const size_t base = (size_t(bg) * a.nsplit + split) * a.Gfull + a.head0;
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      if (h < G) {
        const float v = (KG == 2) ? acc[h] + accs[h * D + dcol] : acc[h];
        a.ws_acc[(base + h) * D + dcol] = v;
        if (dcol == 0) {
          a.ws_ml[(base + h) * 2] = m[h];
          a.ws_ml[(base + h) * 2 + 1] = l[h];
        }
      }
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
  moda_decode_combine_kernel<D><<<unsigned(BG) * a.Gfull, D, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) *why = "decode combine kernel launch failed";
  return e;
}

}  // namespace

DecodeSplit decode_split(const Problem& p) {
  DecodeSplit sp;
  const int nseq = (p.T + kDecKeys - 1) / kDecKeys;
  const int bg = p.B * p.Hkv;
  // at most one wave: one CTA (211 KB of shared memory) per SM of a B200 (148 SMs); a
  // fixed target keeps the workspace size a function of the sizes alone (nsplit <= 148)
  int want = 148 / bg;
  if (want < 1) want = 1;
  if (want > nseq) want = nseq;
  sp.blocks_per_split = (nseq + want - 1) / want;
  sp.nsplit = (nseq + sp.blocks_per_split - 1) / sp.blocks_per_split;  // none empty
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
