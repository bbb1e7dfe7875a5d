// moda_bwd.cu -- MoDA backward for B200 (sm_100a).
//
// The pages define the operator (hyper.ai summary of arXiv 2603.15619, section
// "Mixture-of-Depths Attention (MoDA)": one jointly normalised softmax over the causal
// sequence keys and the query token's own depth keys) but give no backward design.  This
// file computes the exact gradient of that definition given dO, recomputing the softmax
// weights from the forward's log-sum-exp:
//   P = exp(scale*<q,key> - lse),  D = <dO, out>,  dS = P * (<dO, value> - D)
//   dq = scale * sum dS * key;  dk, dkd = scale * sum dS * q;  dv, dvd = sum P * dO.
//
// Three launches:
//  1. moda_bwd_depth_kernel (token-major, CUDA cores, bandwidth-bound): per token of one
//     KV group, D for the G query rows (with -lse*log2e, as the per-tile records the d =
//     128 sequence kernel loads), dkd/dvd for the token's L depth entries, and the depth
//     share of dq, which initialises the fp32 dq accumulator.  Threads split the
//     head dimension into 16-byte column chunks; dot products are finished with warp
//     shuffles, so every depth byte is read from HBM once, with 16-byte coalesced loads.
//  2. moda_bwd_seq_kernel (KV-block-major, tcgen05): one CTA owns 128 sequence keys of
//     one KV head and walks every query tile that sees them.  Per tile the tensor cores
//     compute S^T = K Q^T and dP^T = V dO^T into TMEM; the softmax warps turn them into
//     P^T and dS^T (bf16, back into TMEM, and dS into shared memory); the tensor cores
//     accumulate dV += P^T dO and dK += dS^T Q in TMEM for the whole walk and compute
//     dQ = dS K, which the dQ warps add to the fp32 accumulator: for d = 64 staged in
//     shared memory and added by the TMA unit (bulk tensor reduce-add), for d = 128 (the
//     half-tile variant, 2b) straight from registers with global reductions.
//  3. moda_dq_convert_kernel: dq (bf16) from the fp32 accumulator.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "moda_internal.h"
#include "sm100.cuh"

namespace moda {

namespace {

constexpr int kBwdRegion = 16384;  // one 128-row x 128-byte swizzled region
constexpr float kLog2eBwd = 1.4426950408889634f;

// ============================================================ 1. depth + row terms
constexpr int kDepthThreads = 128;
constexpr int kDepthMaxG = 16;  // heads of one depth-kernel launch (registers hold their dq)
constexpr int kDepthU = 2;     // depth entries per load batch
constexpr int kDepthRing = 8;  // per-thread cp.async ring stages (batches in flight: 7)
constexpr int kDepthRingBytes = kDepthRing * kDepthU * 2 * kDepthThreads * 16;
constexpr int kDepthStageBytes = kDepthRingBytes / 2;  // staged mode: the ring's second half

struct BwdDepthArgs {
  const __nv_bfloat16 *q, *out, *dout, *kd, *vd;
  const float* lse;
  __nv_bfloat16 *dkd, *dvd;
  float* dqacc;  // [B][Hq][T][D] fp32, written (not accumulated) here
  float* drow;   // [B][Hq][T] fp32: D = <dO, out> (null: not written)
  // Row terms of each query tile of the d = 128 sequence kernel, which loads them with one
  // bulk copy per tile: [B*Hkv][nqt][2][128] fp32, record r of tile qt = tile row
  // (t - qt*TQ)*G + head; first -lse*log2(e), then -D*scale.  Rows past the last token or
  // past TQ*G get -inf and 0 (P = 0, dS = 0).  Null: not written.
  float* rt;
  int TQ, nqt;
  long long ntok;  // B * Hkv * T
  int T, L, G;
  // 1 (depth-only attention): the row terms are formed from the depth logits themselves,
  // D = sum_j P_j <dO, vd_j>, in a first pass over the token's entries, instead of from
  // the rounded out.  Every key of such a row is a depth key, so this is the exact D.
  int exact_rows;
  // Set by the launcher for depth-only attention when the kernel keeps q and dO in
  // registers (at most 4 heads) and TPB * L * heads * 8 bytes fit in half the ring: the
  // first pass then stages each entry's (P, <dO, vd>) per head in shared memory, and the
  // gradient pass reads those instead of recomputing them, streaming kd alone.
  int staged;
  // Groups above kDepthMaxG heads run as several launches, one per chunk of at most
  // kDepthMaxG heads: G is this chunk's head count, head0 its first head, Gfull the group
  // size.  dkd/dvd sum over all the group's heads, so the chunks add their contributions
  // into fp32 accumulators in the workspace (acc_mode 1: write, 2: add, 3: add and store
  // the bf16 result); acc_mode 0: the whole group in one launch, bf16 stored directly.
  int head0, Gfull, acc_mode;
  float *dkd_acc, *dvd_acc;  // [B][Hkv][T][L][D] fp32 (acc_mode != 0)
  float scale, scale_log2;
};

// One token slot = D/8 consecutive threads (one 16-byte column chunk each); a CTA works
// on kDepthThreads/(D/8) consecutive tokens of the flattened [B*Hkv][T] token list at a
// time.  The G query rows of the token keep q and dO unpacked to fp32 in registers when
// GM <= 4, else in shared memory (bf16); the dq partial sums of up to GM heads stay in
// registers.
// Butterfly reduce-scatter of the 2*GM partial dot products (y_0..y_{GM-1}, then
// p_0..p_{GM-1}) over the NT lanes of a token slot.  In each round a lane sends half of its
// values to the partner lane (xor o), keeps the other half and adds the partner's copy, so
// the count halves; once a lane holds one value the remaining rounds are plain all-reduce
// steps.  The first round splits the y values from the p values, so the partner across
// the first bit holds p_h for the same heads h.  bf_count: values a lane holds at the end;
// bf_head(lane, i): the head of its i-th value (lanes whose first bit is 0 hold y values).
template <int NT, int NV>
__host__ __device__ constexpr int bf_count() {
  int c = NV;
  for (int o = NT / 2; o > 0 && c > 1; o >>= 1) c /= 2;
  return c;
}
template <int NT, int NV>
__host__ __device__ constexpr int bf_head(int lane, int i) {
  int c = NV, base = 0;
  for (int o = NT / 2; o > 0 && c > 1; o >>= 1) {
    c /= 2;
    if (lane & o) base += c;
  }
  return (base + i) % (NV / 2);
}

// kRT: also write the tiled row-term records (a.rt, the d = 128 sequence kernel's input);
// the instantiation without them is the one depth-only attention and d = 64 run.
template <int D, int GM, bool kRT>
// (GM <= 4: at most 168 registers, three CTAs per SM; measured faster than 188 registers
// and two CTAs)
__global__ void __launch_bounds__(kDepthThreads, GM <= 4 ? 3 : 1)
    moda_bwd_depth_kernel(const BwdDepthArgs a) {
  constexpr int NT = D / 8;
  constexpr int TPB = kDepthThreads / NT;
  extern __shared__ __align__(16) uint8_t dsm[];
  const int tid = threadIdx.x;
  const int slot = tid / NT, cs = tid % NT;
  const int G = a.G;
  constexpr bool kReg = GM <= 4;  // q, dO of the token's heads held in registers
  const uint32_t q_s = smem_u32(dsm) + uint32_t(slot * 2 * G * D * 2);
  const uint32_t do_s = q_s + uint32_t(G * D * 2);
  // Per-thread ring of depth-entry chunks filled by cp.async, kDNS batches of kU entries
  // (kd and vd) deep, after the q/dO slots (none when they live in registers): each thread
  // copies and reads back only its own 16-byte chunks, so no barrier is involved.
  constexpr int kU = kDepthU;
  constexpr int kDNS = kDepthRing;
  const uint32_t ring = smem_u32(dsm) + (kReg ? 0u : uint32_t(TPB * 2 * G * D * 2));
  auto rslot = [&](int stg, int u, int kv) {
    return ring + uint32_t((((stg * kU + u) * 2 + kv) * kDepthThreads + tid) * 16);
  };
  const long long L = a.L;
  // Staged depth-only attention (see BwdDepthArgs::staged): the ring's first half carries
  // kd alone, its second half holds each token's [L][GM] (P, <dO, vd>) pairs.
  constexpr bool kCanStage = !kRT && kReg;
  const bool staged = kCanStage && a.staged != 0;
  auto rslot_kd = [&](int stg, int u) {
    return ring + uint32_t(((stg * kU + u) * kDepthThreads + tid) * 16);
  };
  const uint32_t stage_slot =
      ring + uint32_t(kDepthStageBytes) + uint32_t(slot) * uint32_t(L) * uint32_t(GM * 8);

  for (long long base = (long long)blockIdx.x * TPB; base < a.ntok;
       base += (long long)gridDim.x * TPB) {
    const long long tk = base + slot;
    const bool valid = tk < a.ntok;
    const long long tkc = valid ? tk : a.ntok - 1;
    const long long bg = tkc / a.T;
    const int t = int(tkc - bg * a.T);
    const int qt = kRT ? t / a.TQ : 0, tq = t - qt * a.TQ;
    float* const rt_tile = kRT ? a.rt + ((bg * a.nqt + qt) << 8) : nullptr;
    const int r0 = tq * a.Gfull + a.head0;  // tile row of this chunk's head 0

    float lse2[GM], drw[GM];
    float qreg[kReg ? GM : 1][8], dreg[kReg ? GM : 1][8];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      lse2[h] = 0.f;
      drw[h] = 0.f;
      if constexpr (kReg) {
#pragma unroll
        for (int e = 0; e < 8; ++e) qreg[h][e] = dreg[h][e] = 0.f;
      }
      if (h < G) {
        const long long row = (bg * a.Gfull + a.head0 + h) * a.T + t;
        float part = 0.f;
        if (valid) {
          const uint4 qw = ldg_nc_v4(a.q + row * D + cs * 8);
          const uint4 dw = ldg_nc_v4(a.dout + row * D + cs * 8);
          const uint4 ow = ldg_nc_v4(a.out + row * D + cs * 8);
          float df[8], of[8];
          unpack8(dw, df);
          unpack8(ow, of);
          if constexpr (kReg) {
            unpack8(qw, qreg[h]);
#pragma unroll
            for (int e = 0; e < 8; ++e) dreg[h][e] = df[e];
          } else {
            sts128(q_s + uint32_t((h * D + cs * 8) * 2), qw);
            sts128(do_s + uint32_t((h * D + cs * 8) * 2), dw);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) part = fmaf(df[e], of[e], part);
          lse2[h] = a.lse[row] * kLog2eBwd;
        }
#pragma unroll
        for (int o = NT / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        drw[h] = part;
        if (valid && cs == 0 && a.drow) a.drow[row] = part;
        if (kRT && valid && cs == (h & (NT - 1))) {
          rt_tile[r0 + h] = -lse2[h];
          rt_tile[128 + r0 + h] = -part * a.scale;
        }
      }
    }
    // the last token of a tile fills the tile's records past its rows (once, in the first
    // head chunk)
    if (kRT && valid && a.head0 == 0 && (tq == a.TQ - 1 || t == a.T - 1)) {
      for (int r = r0 + a.Gfull + cs; r < 128; r += NT) {
        rt_tile[r] = -INFINITY;
        rt_tile[128 + r] = 0.f;
      }
    }
    __syncwarp();

    float dq[GM][8];
#pragma unroll
    for (int h = 0; h < GM; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) dq[h][e] = 0.f;

    const long long tok_off = (bg * a.T + t) * L * D + cs * 8;
    // (depth-only attention only: the d = 128 MoDA instantiation, with its row-term
    // records, never takes this path and is compiled without it)
    if constexpr (!kRT) {
      if (a.exact_rows) {
        // D_h = sum_j P_hj <dO_h, vd_j>, P_hj = 2^(y_hj * scale * log2(e) - lse_h * log2(e)):
        // the weights the gradient pass uses, which it reads back from the staged pairs or
        // (not staged) recomputes, reading kd and vd once more.  The dot products are
        // finished by the same butterfly as the gradient pass's (below), each lane summing
        // P * p for the heads it ends up holding; one broadcast per token.
        constexpr int kNV0 = 2 * GM, kBC0 = bf_count<NT, kNV0>();
        float lse_mine[kBC0], dsum[kBC0];
#pragma unroll
        for (int i = 0; i < kBC0; ++i) {
          lse_mine[i] = dsum[i] = 0.f;
#pragma unroll
          for (int h = 0; h < GM; ++h)
            if (h == bf_head<NT, kNV0>(cs, i)) lse_mine[i] = lse2[h];
        }
        const bool is_y = (cs & (NT / 2)) == 0;
        // one entry of the first pass: the dot products, their butterfly, P and the row term
        auto pre_entry = [&](const long long j, const uint4 kw, const uint4 vw) {
          float kf[8], vf[8];
          unpack8(kw, kf);
          unpack8(vw, vf);
          float bv[kNV0];
#pragma unroll
          for (int h = 0; h < GM; ++h) {
            bv[h] = bv[GM + h] = 0.f;
            if (h < G) {
              float qf[8], df[8];
              if constexpr (kReg) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  qf[e] = qreg[h][e];
                  df[e] = dreg[h][e];
                }
              } else {
                unpack8(lds128(q_s + uint32_t((h * D + cs * 8) * 2)), qf);
                unpack8(lds128(do_s + uint32_t((h * D + cs * 8) * 2)), df);
              }
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                bv[h] = fmaf(qf[e], kf[e], bv[h]);
                bv[GM + h] = fmaf(df[e], vf[e], bv[GM + h]);
              }
            }
          }
          int c = kNV0;
#pragma unroll
          for (int o = NT / 2; o > 0; o >>= 1) {
            if (c > 1) {
              const bool up = (cs & o) != 0;
#pragma unroll
              for (int i = 0; i < kNV0 / 2; ++i) {
                if (i < c / 2) {
                  const float send = up ? bv[i] : bv[c / 2 + i];
                  const float keep = up ? bv[c / 2 + i] : bv[i];
                  bv[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
              }
              c /= 2;
            } else {
              bv[0] += __shfl_xor_sync(0xffffffffu, bv[0], o);
            }
          }
#pragma unroll
          for (int i = 0; i < kBC0; ++i) {
            const float other = __shfl_xor_sync(0xffffffffu, bv[i], NT / 2);
            const float yy = is_y ? bv[i] : other, pp = is_y ? other : bv[i];
            const float Pw = ex2(yy * a.scale_log2 - lse_mine[i]);
            dsum[i] = fmaf(Pw, pp, dsum[i]);
            if constexpr (kCanStage) {
              // one lane per head writes: a y lane whose all-reduce bits are 0 (lanes that
              // differ only in those bits hold the same sums)
              constexpr int kDup = NT / kNV0 - 1;
              if (staged && is_y && (cs & kDup) == 0)
                sts64f(stage_slot + uint32_t((j * GM + bf_head<NT, kNV0>(cs, i)) * 8), Pw, pp);
            }
          }
        };
        // kd and vd stream through a cp.async ring: staged, a four-stage one in the first
        // half of the ring memory (the gradient pass reuses it for kd alone once this pass
        // has drained); otherwise the whole ring, which the gradient pass then refills
        auto pre_ring = [&](auto stages_c, auto slot_fn) {
          constexpr int kPS = decltype(stages_c)::value;
          auto issue_pre = [&](long long b) {
            const int stg = int(b % kPS);
#pragma unroll
            for (int u = 0; u < kU; ++u) {
              const long long j = b * kU + u;
              if (valid && j < L) {
                cp_async16(slot_fn(stg, u, 0), a.kd + tok_off + j * D);
                cp_async16(slot_fn(stg, u, 1), a.vd + tok_off + j * D);
              }
            }
            cp_async_commit();
          };
#pragma unroll
          for (int b = 0; b < kPS - 1; ++b) issue_pre(b);
          for (long long j0 = 0; j0 < L; j0 += kU) {
            const long long b = j0 / kU;
            issue_pre(b + kPS - 1);
            cp_async_wait<kPS - 1>();  // batch b has landed
            const int stg = int(b % kPS);
#pragma unroll
            for (int u = 0; u < kU; ++u) {
              if (j0 + u >= L) break;
              uint4 kw = make_uint4(0, 0, 0, 0), vw = make_uint4(0, 0, 0, 0);
              if (valid) {
                kw = lds128(slot_fn(stg, u, 0));
                vw = lds128(slot_fn(stg, u, 1));
              }
              pre_entry(j0 + u, kw, vw);
            }
          }
          cp_async_wait<0>();  // (only empty groups remain) before the ring is reused
        };
        if (staged) {
          if constexpr (kCanStage) {
            auto rslot_pre = [&](int stg, int u, int kv) {
              return ring + uint32_t((((stg * kU + u) * 2 + kv) * kDepthThreads + tid) * 16);
            };
            pre_ring(std::integral_constant<int, 4>{}, rslot_pre);
          }
        } else {
          pre_ring(std::integral_constant<int, kDNS>{}, rslot);
        }
        const int slot0 = (threadIdx.x & 31) & ~(NT - 1);
#pragma unroll
        for (int h = 0; h < GM; ++h) {
          int src = 0, si = 0;
#pragma unroll
          for (int l2 = NT / 2 - 1; l2 >= 0; --l2)
#pragma unroll
            for (int i = 0; i < kBC0; ++i)
              if (bf_head<NT, kNV0>(l2, i) == h) { src = l2; si = i; }
          const float dh = __shfl_sync(0xffffffffu, dsum[si], slot0 + src);
          if (h < G) {
            drw[h] = dh;
            if (valid && cs == 0 && a.drow) a.drow[(bg * a.Gfull + a.head0 + h) * a.T + t] = dh;
          }
        }
        if (staged) __syncwarp();  // the staged pairs, written by some lanes, read by all
      }
    }
    // (after the exact row terms above, when they apply) row terms of the heads whose P and
    // dS this lane computes (see the butterfly below)
    constexpr int kNV = 2 * GM, kBC = bf_count<NT, kNV>();
    float my_lse2[kBC], my_drw[kBC];
#pragma unroll
    for (int i = 0; i < kBC; ++i) {
      my_lse2[i] = my_drw[i] = 0.f;
#pragma unroll
      for (int h = 0; h < GM; ++h)
        if (h == bf_head<NT, kNV>(cs, i) % GM) {
          my_lse2[i] = lse2[h];
          my_drw[i] = drw[h];
        }
    }
    if (staged) {
      if constexpr (kCanStage) {
        // gradient pass over the staged pairs: kd streams alone through the ring's first
        // half, P and <dO, vd> of every head come from shared memory, dS = P (p - D)
        auto issue_kd = [&](long long b) {
          const int stg = int(b % kDNS);
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const long long j = b * kU + u;
            if (valid && j < L) cp_async16(rslot_kd(stg, u), a.kd + tok_off + j * D);
          }
          cp_async_commit();
        };
#pragma unroll
        for (int b = 0; b < kDNS - 1; ++b) issue_kd(b);
        for (long long j0 = 0; j0 < L; j0 += kU) {
          const long long b = j0 / kU;
          issue_kd(b + kDNS - 1);
          cp_async_wait<kDNS - 1>();  // batch b has landed
          const int stg = int(b % kDNS);
          uint4 kwu[kU];
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            kwu[u] = make_uint4(0, 0, 0, 0);
            if (valid && j0 + u < L) kwu[u] = lds128(rslot_kd(stg, u));
          }
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            if (j0 + u >= L) break;
            const long long j = j0 + u;
            float kf[8];
            unpack8(kwu[u], kf);
            float dv[8], dk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) dv[e] = dk[e] = 0.f;
#pragma unroll
            for (int h = 0; h < GM; ++h) {
              if (h < G) {
                const float2 Pp = lds64f(stage_slot + uint32_t((j * GM + h) * 8));
                const float2 P2 = make_float2(Pp.x, Pp.x);
                const float dSv = Pp.x * (Pp.y - drw[h]);
                const float2 dS2 = make_float2(dSv, dSv);
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                  const float2 v2 = ffma2(P2, make_float2(dreg[h][e], dreg[h][e + 1]),
                                          make_float2(dv[e], dv[e + 1]));
                  const float2 k2 = ffma2(dS2, make_float2(qreg[h][e], qreg[h][e + 1]),
                                          make_float2(dk[e], dk[e + 1]));
                  const float2 q2 = ffma2(dS2, make_float2(kf[e], kf[e + 1]),
                                          make_float2(dq[h][e], dq[h][e + 1]));
                  dv[e] = v2.x; dv[e + 1] = v2.y;
                  dk[e] = k2.x; dk[e + 1] = k2.y;
                  dq[h][e] = q2.x; dq[h][e + 1] = q2.y;
                }
              }
            }
            if (valid) {  // (one launch holds the whole group here: acc_mode 0)
              const long long o = tok_off + j * D;
              *reinterpret_cast<uint4*>(a.dvd + o) = pack8(dv, 1.f);
              *reinterpret_cast<uint4*>(a.dkd + o) = pack8(dk, a.scale);
            }
          }
        }
        cp_async_wait<0>();  // (only empty groups remain) before the ring is reused
      }
    } else {
    const long long nbat = (L + kU - 1) / kU;
    // batch b's copies (an empty group past the last batch keeps the group count uniform)
    auto issue = [&](long long b) {
      const int stg = int(b % kDNS);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const long long j = b * kU + u;
        if (valid && j < L) {
          cp_async16(rslot(stg, u, 0), a.kd + tok_off + j * D);
          cp_async16(rslot(stg, u, 1), a.vd + tok_off + j * D);
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int b = 0; b < kDNS - 1; ++b) issue(b);
    for (long long j0 = 0; j0 < L; j0 += kU) {
      const long long b = j0 / kU;
      issue(b + kDNS - 1);
      cp_async_wait<kDNS - 1>();  // batch b has landed
      const int stg = int(b % kDNS);
      uint4 kwu[kU], vwu[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        kwu[u] = vwu[u] = make_uint4(0, 0, 0, 0);
        if (valid && j0 + u < L) {
          kwu[u] = lds128(rslot(stg, u, 0));
          vwu[u] = lds128(rslot(stg, u, 1));
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
      if (j0 + u >= L) break;
      const long long j = j0 + u;
      float kf[8], vf[8];
      unpack8(kwu[u], kf);
      unpack8(vwu[u], vf);
      float y[GM], p[GM];
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        y[h] = 0.f;
        p[h] = 0.f;
        if (h < G) {
          float qf[8], df[8];
          if constexpr (kReg) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              qf[e] = qreg[h][e];
              df[e] = dreg[h][e];
            }
          } else {
            unpack8(lds128(q_s + uint32_t((h * D + cs * 8) * 2)), qf);
            unpack8(lds128(do_s + uint32_t((h * D + cs * 8) * 2)), df);
          }
          // packed pairs: one f32x2 FMA per two products
          float2 y2 = make_float2(0.f, 0.f), p2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            y2 = ffma2(make_float2(qf[e], qf[e + 1]), make_float2(kf[e], kf[e + 1]), y2);
            p2 = ffma2(make_float2(df[e], df[e + 1]), make_float2(vf[e], vf[e + 1]), p2);
          }
          y[h] = y2.x + y2.y;
          p[h] = p2.x + p2.y;
        }
      }
      // finish the token's dot products: butterfly reduce-scatter over the slot's lanes
      float bv[kNV];
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        bv[h] = y[h];
        bv[GM + h] = p[h];
      }
      {
        int c = kNV;
#pragma unroll
        for (int o = NT / 2; o > 0; o >>= 1) {
          if (c > 1) {
            const bool up = (cs & o) != 0;
#pragma unroll
            for (int i = 0; i < kNV / 2; ++i) {
              if (i < c / 2) {
                const float send = up ? bv[i] : bv[c / 2 + i];
                const float keep = up ? bv[c / 2 + i] : bv[i];
                bv[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
              }
            }
            c /= 2;
          } else {
            bv[0] += __shfl_xor_sync(0xffffffffu, bv[0], o);
          }
        }
      }
      // bv[0..kBC) are now full sums; the partner across the first bit holds the other
      // kind (y or p) of the same heads: P and dS of those heads, then broadcast
      float bP[kBC], bS[kBC];
      {
        const bool is_y = (cs & (NT / 2)) == 0;
#pragma unroll
        for (int i = 0; i < kBC; ++i) {
          const float other = __shfl_xor_sync(0xffffffffu, bv[i], NT / 2);
          const float yy = is_y ? bv[i] : other, pp = is_y ? other : bv[i];
          bP[i] = ex2(yy * a.scale_log2 - my_lse2[i]);
          bS[i] = bP[i] * (pp - my_drw[i]);
        }
      }
      const int slot0 = (threadIdx.x & 31) & ~(NT - 1);  // first lane of this token slot
      float dv[8], dk[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) dv[e] = dk[e] = 0.f;
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        if (h < G) {
          // the value of head h sits in slot i of the y lanes l with bf_head(l, i) == h
          int src = 0, si = 0;
#pragma unroll
          for (int l2 = NT / 2 - 1; l2 >= 0; --l2)
#pragma unroll
            for (int i = 0; i < kBC; ++i)
              if (bf_head<NT, kNV>(l2, i) == h) { src = l2; si = i; }
          const float P = __shfl_sync(0xffffffffu, bP[si], slot0 + src);
          const float dS = __shfl_sync(0xffffffffu, bS[si], slot0 + src);
          float qf[8], df[8];
          if constexpr (kReg) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              qf[e] = qreg[h][e];
              df[e] = dreg[h][e];
            }
          } else {
            unpack8(lds128(q_s + uint32_t((h * D + cs * 8) * 2)), qf);
            unpack8(lds128(do_s + uint32_t((h * D + cs * 8) * 2)), df);
          }
          const float2 P2 = make_float2(P, P), dS2 = make_float2(dS, dS);
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const float2 v2 = ffma2(P2, make_float2(df[e], df[e + 1]),
                                    make_float2(dv[e], dv[e + 1]));
            const float2 k2 = ffma2(dS2, make_float2(qf[e], qf[e + 1]),
                                    make_float2(dk[e], dk[e + 1]));
            const float2 q2 = ffma2(dS2, make_float2(kf[e], kf[e + 1]),
                                    make_float2(dq[h][e], dq[h][e + 1]));
            dv[e] = v2.x; dv[e + 1] = v2.y;
            dk[e] = k2.x; dk[e + 1] = k2.y;
            dq[h][e] = q2.x; dq[h][e + 1] = q2.y;
          }
        }
      }
      if (valid) {
        const long long o = tok_off + j * D;
        if (a.acc_mode == 0) {
          *reinterpret_cast<uint4*>(a.dvd + o) = pack8(dv, 1.f);
          *reinterpret_cast<uint4*>(a.dkd + o) = pack8(dk, a.scale);
        } else {
          // this chunk's heads' share, summed with the other chunks' in fp32
          float4* av = reinterpret_cast<float4*>(a.dvd_acc + o);
          float4* ak = reinterpret_cast<float4*>(a.dkd_acc + o);
          if (a.acc_mode != 1) {
            const float4 v0 = av[0], v1 = av[1], k0 = ak[0], k1 = ak[1];
            dv[0] += v0.x; dv[1] += v0.y; dv[2] += v0.z; dv[3] += v0.w;
            dv[4] += v1.x; dv[5] += v1.y; dv[6] += v1.z; dv[7] += v1.w;
            dk[0] += k0.x; dk[1] += k0.y; dk[2] += k0.z; dk[3] += k0.w;
            dk[4] += k1.x; dk[5] += k1.y; dk[6] += k1.z; dk[7] += k1.w;
          }
          if (a.acc_mode == 3) {
            *reinterpret_cast<uint4*>(a.dvd + o) = pack8(dv, 1.f);
            *reinterpret_cast<uint4*>(a.dkd + o) = pack8(dk, a.scale);
          } else {
            av[0] = make_float4(dv[0], dv[1], dv[2], dv[3]);
            av[1] = make_float4(dv[4], dv[5], dv[6], dv[7]);
            ak[0] = make_float4(dk[0], dk[1], dk[2], dk[3]);
            ak[1] = make_float4(dk[4], dk[5], dk[6], dk[7]);
          }
        }
      }
      }
    }
    cp_async_wait<0>();  // (only empty groups remain) before the ring is reused
    (void)nbat;
    }
    if (valid) {
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        if (h < G) {
          const long long row = (bg * a.Gfull + a.head0 + h) * a.T + t;
          float4* dst = reinterpret_cast<float4*>(a.dqacc + row * D + cs * 8);
          dst[0] = make_float4(dq[h][0] * a.scale, dq[h][1] * a.scale, dq[h][2] * a.scale,
                               dq[h][3] * a.scale);
          dst[1] = make_float4(dq[h][4] * a.scale, dq[h][5] * a.scale, dq[h][6] * a.scale,
                               dq[h][7] * a.scale);
        }
      }
    }
    __syncwarp();  // the slot's q/dO copies are rewritten by the next pass
  }
}

// ============================================================ 2. sequence part
constexpr int kSeqThreads = 320;  // warps 0-3 P/dS, 4-7 dQ, 8 TMA, 9 tcgen05

template <int D>
struct SeqCfg {
  static constexpr int kRegions = D / 64;
  static constexpr int kTile = kRegions * kBwdRegion;  // 128 rows x D bf16, swizzled
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTile;
  static constexpr int kOffQ = 2 * kTile;   // two stages
  static constexpr int kOffDO = 4 * kTile;  // two stages
  static constexpr int kOffDS = 6 * kTile;  // dS, 128 rows x 128 keys bf16, MN-major
  static constexpr int kOffLD = kOffDS + 2 * kBwdRegion;  // [2 stages][lse2 | D][128] f32
  static constexpr int kOffBar = kOffLD + 2 * 2 * 128 * 4;
  static constexpr int kSmemBytes = kOffBar + 256;
};

struct SeqBars {
  uint64_t kv_full;
  uint64_t q_full[2], q_empty[2];
  uint64_t do_full[2], do_empty[2];
  uint64_t s_full, dp_full, pds_full, dq_full, dq_free, kv_done;
  uint32_t tmem_base;
  int abort;
};

struct SeqArgs {
  __nv_bfloat16 *dk, *dv;
  float* dqacc;
  const float *lse, *drow;  // d = 64 kernel: [B][Hq][T] each
  const float* rt;          // d = 128 kernel: tiled row terms (BwdDepthArgs::rt)
  int Hkv, T, G, TQ, nqt, BG, causal;
  float scale, scale_log2;
};

template <int D>
__global__ void __launch_bounds__(kSeqThreads, 1)
    moda_bwd_seq_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmDO,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmDQ, const SeqArgs a) {
  using Cfg = SeqCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  // The swizzled operand layouts need a 1024-byte aligned base, and there is no room
  // to realign inside the shared-memory budget: refuse to run otherwise.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicOr(&g_error_word, kErrInternal);
    return;
  }
  const uint32_t s0 = smem_u32(smem);
  const uint32_t sK = s0 + Cfg::kOffK, sV = s0 + Cfg::kOffV, sDS = s0 + Cfg::kOffDS;
  auto sQ = [&](int st) { return s0 + Cfg::kOffQ + uint32_t(st) * Cfg::kTile; };
  auto sDO = [&](int st) { return s0 + Cfg::kOffDO + uint32_t(st) * Cfg::kTile; };
  float* ld_s = reinterpret_cast<float*>(smem + Cfg::kOffLD);
  SeqBars* bars = reinterpret_cast<SeqBars*>(smem + Cfg::kOffBar);
  volatile int* abort_flag = &bars->abort;
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };

  const int warp = threadIdx.x >> 5;
  const int bg = blockIdx.x % a.BG;
  const int kb = blockIdx.x / a.BG;  // key blocks nearest the start see the most tiles
  const int key0 = kb * 128;
  const int first_qt = a.causal ? key0 / a.TQ : 0;
  const int ntiles = a.nqt - first_qt;

  if (threadIdx.x == 0) {
    mbar_init(bar(bars->kv_full), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(bars->q_full[i]), 1);
      mbar_init(bar(bars->q_empty[i]), 1);
      mbar_init(bar(bars->do_full[i]), 1);
      mbar_init(bar(bars->do_empty[i]), 1);
    }
    mbar_init(bar(bars->s_full), 1);
    mbar_init(bar(bars->dp_full), 1);
    mbar_init(bar(bars->pds_full), 128);
    mbar_init(bar(bars->dq_full), 1);
    mbar_init(bar(bars->dq_free), 128);
    mbar_init(bar(bars->kv_done), 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  // Q/dO rows past TQ*G (G not dividing 128) never receive TMA data: zero them once.
  if (threadIdx.x < 128 && threadIdx.x >= a.TQ * a.G) {
    for (int st = 0; st < 2; ++st)
      for (int rg = 0; rg < Cfg::kRegions; ++rg) {
        uint4* rq = reinterpret_cast<uint4*>(smem + Cfg::kOffQ + st * Cfg::kTile +
                                             rg * kBwdRegion + threadIdx.x * 128);
        uint4* rd = reinterpret_cast<uint4*>(smem + Cfg::kOffDO + st * Cfg::kTile +
                                             rg * kBwdRegion + threadIdx.x * 128);
        for (int c = 0; c < 8; ++c) rq[c] = rd[c] = make_uint4(0, 0, 0, 0);
      }
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // TMEM columns: S^T/P^T and then dQ [0,128), dP^T/dS^T [128,256), dV [256,256+D),
  // dK [256+D, 256+2D).  P^T and dS^T are stored as bf16 hi/lo pairs: each 32-row chunk
  // occupies 32 columns, 16 of packed hi values then 16 of packed lo values.
  const uint32_t tS = tmem, tDP = tmem + 128, tDV = tmem + 256, tDK = tmem + 256 + D;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmDO);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(bar(bars->kv_full), 2 * Cfg::kTile);
      for (int rg = 0; rg < Cfg::kRegions; ++rg) {
        tma_load_3d(sK + rg * kBwdRegion, &tmK, bar(bars->kv_full), rg * 64, key0, bg);
        tma_load_3d(sV + rg * kBwdRegion, &tmV, bar(bars->kv_full), rg * 64, key0, bg);
      }
      const uint32_t qbytes = Cfg::kRegions * 128 * a.G * a.TQ;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i & 1;
        const int t0 = (first_qt + i) * a.TQ;
        if (i >= 2) mbar_wait(bar(bars->q_empty[st]), ((i >> 1) - 1) & 1, abort_flag);
        mbar_expect_tx(bar(bars->q_full[st]), qbytes);
        for (int rg = 0; rg < Cfg::kRegions; ++rg)
          tma_load_4d(sQ(st) + rg * kBwdRegion, &tmQ, bar(bars->q_full[st]), rg * 64, 0, t0,
                      bg);
        if (i >= 2) mbar_wait(bar(bars->do_empty[st]), ((i >> 1) - 1) & 1, abort_flag);
        mbar_expect_tx(bar(bars->do_full[st]), qbytes);
        for (int rg = 0; rg < Cfg::kRegions; ++rg)
          tma_load_4d(sDO(st) + rg * kBwdRegion, &tmDO, bar(bars->do_full[st]), rg * 64, 0,
                      t0, bg);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ tcgen05 issuer
    if (elect_one()) {
      constexpr uint32_t idesc_t = make_idesc_bf16(128, 128, 0, 0);  // S^T, dP^T
      constexpr uint32_t idesc_g = make_idesc_bf16(128, D, 0, 1);    // dV, dK (A in TMEM)
      constexpr uint32_t idesc_q = make_idesc_bf16(128, D, 1, 1);    // dQ (A = dS, MN-major)
      mbar_wait(bar(bars->kv_full), 0, abort_flag);
      // S^T(i) = K Q(i)^T and dP^T(i) = V dO(i)^T
      auto issue_s = [&](int i) {
        mbar_wait(bar(bars->q_full[i & 1]), (i >> 1) & 1, abort_flag);
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks / 4) * kBwdRegion + (ks % 4) * 32;
          mma_ss(tS, make_sdesc_sw128(sK + off, 16, 1024),
                 make_sdesc_sw128(sQ(i & 1) + off, 16, 1024), idesc_t, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(bars->s_full));
      };
      auto issue_dp = [&](int i) {
        mbar_wait(bar(bars->do_full[i & 1]), (i >> 1) & 1, abort_flag);
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks / 4) * kBwdRegion + (ks % 4) * 32;
          mma_ss(tDP, make_sdesc_sw128(sV + off, 16, 1024),
                 make_sdesc_sw128(sDO(i & 1) + off, 16, 1024), idesc_t, ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(bars->dp_full));
      };
      // Per tile: dV, then dQ into the S^T columns (free once dV has read P^T), then dK,
      // then the next tile's dP^T (its columns are free once dK has read dS^T).  Only
      // the next S^T waits for the dQ readout, which overlaps dK and the next dP^T.
      issue_s(0);
      issue_dp(0);
      for (int i = 0; i < ntiles; ++i) {
        const int st = i & 1;
        mbar_wait(bar(bars->pds_full), i & 1, abort_flag);
        tc_fence_after();
        // dV += P^T dO : A = P^T (TMEM, keys x rows; hi then lo), B = dO (rows x D, MN-major).
        // K-step ks covers rows 16ks..16ks+15: packed columns 32(ks/2) + 8(ks%2), lo +16.
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t col = (ks >> 1) * 32 + (ks & 1) * 8;
          const uint64_t bd = make_sdesc_sw128(sDO(st) + ks * 2048, kBwdRegion, 1024);
          mma_ts(tDV, tS + col, bd, idesc_g, (i > 0 || ks > 0) ? 1u : 0u);
          mma_ts(tDV, tS + col + 16, bd, idesc_g, 1u);
        }
        tc_commit(bar(bars->do_empty[st]));
        // dQ = dS K into the S^T columns : A = dS (rows x keys, MN-major in shared memory),
        // B = K (keys x D)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tS, make_sdesc_sw128(sDS + ks * 2048, kBwdRegion, 1024),
                 make_sdesc_sw128(sK + ks * 2048, kBwdRegion, 1024), idesc_q, ks > 0 ? 1u : 0u);
        tc_commit(bar(bars->dq_full));
        // dK += dS^T Q (hi then lo)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t col = (ks >> 1) * 32 + (ks & 1) * 8;
          const uint64_t bd = make_sdesc_sw128(sQ(st) + ks * 2048, kBwdRegion, 1024);
          mma_ts(tDK, tDP + col, bd, idesc_g, (i > 0 || ks > 0) ? 1u : 0u);
          mma_ts(tDK, tDP + col + 16, bd, idesc_g, 1u);
        }
        tc_commit(bar(bars->q_empty[st]));
        if (i + 1 < ntiles) {
          issue_dp(i + 1);
          mbar_wait(bar(bars->dq_free), i & 1, abort_flag);
          issue_s(i + 1);
        }
      }
      tc_commit(bar(bars->kv_done));
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ P / dS warps
    const int tid = threadIdx.x;  // TMEM lane = key key0 + tid
    const int key = key0 + tid;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const int hl = tid % a.G, tok = tid / a.G;
    // lse and D of row `tid` of tile i, loaded one tile ahead so the global-load latency
    // stays off the per-tile critical path
    auto load_rowterms = [&](int i, float& lse2v, float& dv_) {
      const int t = (first_qt + i) * a.TQ + tok;
      const bool valid = i < ntiles && tok < a.TQ && t < a.T;
      const long long idx = ((long long)bg * a.G + hl) * a.T + (valid ? t : 0);
      lse2v = valid ? -a.lse[idx] * kLog2eBwd : -INFINITY;  // stored negated
      dv_ = valid ? -a.drow[idx] : 0.f;                      // stored negated
    };
    float nxt_lse, nxt_d;
    load_rowterms(0, nxt_lse, nxt_d);
    for (int i = 0; i < ntiles; ++i) {
      const int qt = first_qt + i;
      const int b = i & 1;
      ld_s[b * 256 + tid] = nxt_lse;
      ld_s[b * 256 + 128 + tid] = nxt_d;
      named_bar_sync(1, 128);
      load_rowterms(i + 1, nxt_lse, nxt_d);
      // rows r < r_min hold tokens before this key (causal) -- their weight is zero
      int r_min = 0;
      if (key >= a.T)
        r_min = 1 << 30;
      else if (a.causal)
        r_min = a.G * (key - qt * a.TQ);
      const float* nlse2 = ld_s + b * 256;      // -lse * log2e per row
      const float* ndr = ld_s + b * 256 + 128;  // -D per row
      mbar_wait(bar(bars->s_full), i & 1, abort_flag);
      mbar_wait(bar(bars->dp_full), i & 1, abort_flag);
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t s[32], dp[32];
        tmem_ld32(tS + lane_base + c * 32, s);
        tmem_ld32(tDP + lane_base + c * 32, dp);
        tmem_wait_ld();
        // P and dS as bf16 pairs hi + lo (lo = what bf16 rounding dropped): the dV and dK
        // products use both, so their operands carry about 2^-17 relative error instead
        // of 2^-9.  Chunk c writes its 32 columns back over the 32 it read: hi in the
        // first 16, lo in the last 16.
        uint32_t pp[16], pl[16], pd[16], dl[16];
        const bool masked = r_min > c * 32;  // some row of this chunk precedes the key
        const float2 sl2 = make_float2(a.scale_log2, a.scale_log2);
        const float2 sc2 = make_float2(a.scale, a.scale);
        const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int r = c * 32 + e;
          // P = 2^(s*scale*log2e - lse*log2e); the row terms are stored negated
          const float2 arg = ffma2(make_float2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])),
                                   sl2, make_float2(nlse2[r], nlse2[r + 1]));
          float P0 = ex2(arg.x), P1 = ex2(arg.y);
          if (masked) {
            if (r < r_min) P0 = 0.f;
            if (r + 1 < r_min) P1 = 0.f;
          }
          // dS = P * scale * (dP - D)
          const float2 Ps = fmul2(make_float2(P0, P1), sc2);
          const float2 dd = fadd2(make_float2(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])),
                                  make_float2(ndr[r], ndr[r + 1]));
          const float2 dS = fmul2(Ps, dd);
          const uint32_t ph = pack_bf16x2(P0, P1), dh = pack_bf16x2(dS.x, dS.y);
          const float2 plo = ffma2(make_float2(bf16lo(ph), bf16hi(ph)), neg1, make_float2(P0, P1));
          const float2 dlo = ffma2(make_float2(bf16lo(dh), bf16hi(dh)), neg1, dS);
          pp[e / 2] = ph;
          pl[e / 2] = pack_bf16x2(plo.x, plo.y);
          pd[e / 2] = dh;
          dl[e / 2] = pack_bf16x2(dlo.x, dlo.y);
        }
        tmem_st16(tS + lane_base + c * 32, pp);
        tmem_st16(tS + lane_base + c * 32 + 16, pl);
        tmem_st16(tDP + lane_base + c * 32, pd);
        tmem_st16(tDP + lane_base + c * 32 + 16, dl);
        // dS row-block for the dQ product: rows c*32..c*32+31 of this key's column
        const uint32_t reg = sDS + (c >> 1) * kBwdRegion + uint32_t(tid) * 128;
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          const uint32_t chunk = (c & 1) * 4 + qd;
          sts128(reg + ((chunk ^ (tid & 7)) << 4),
                 make_uint4(pd[qd * 4], pd[qd * 4 + 1], pd[qd * 4 + 2], pd[qd * 4 + 3]));
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(bars->pds_full));
    }
    // epilogue: dV, dK rows of this key
    mbar_wait(bar(bars->kv_done), 0, abort_flag);
    tc_fence_after();
    const bool kvalid = key < a.T;
    const long long koff = ((long long)bg * a.T + (kvalid ? key : 0)) * D;
#pragma unroll 1
    for (int which = 0; which < 2; ++which) {
      const uint32_t tsrc = (which ? tDK : tDV) + lane_base;
      __nv_bfloat16* dst = (which ? a.dk : a.dv) + koff;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tsrc + cc * 32, o);
        tmem_wait_ld();
        if (kvalid) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(o[v * 8 + e]);
            d4[v] = pack8(f, 1.f);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ dQ warps 4-7
    // dQ of each tile is added to the fp32 accumulator by the TMA unit: the warps stage
    // it, 64 columns at a time, as two 128B-swizzled fp32 regions in the dS buffer (idle
    // from the dQ product's completion until the next tile's P/dS) and one thread issues
    // the bulk tensor reduce-adds.
    const int r = threadIdx.x - 128;  // TMEM lane = tile row
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    for (int i = 0; i < ntiles; ++i) {
      const int t0q = (first_qt + i) * a.TQ;
      mbar_wait(bar(bars->dq_full), i & 1, abort_flag);
      tc_fence_after();
#pragma unroll 1
      for (int half = 0; half < D / 64; ++half) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t o[32];
          tmem_ld32(tS + lane_base + half * 64 + q * 32, o);
          tmem_wait_ld();
          const uint32_t reg = sDS + q * kBwdRegion + uint32_t(r) * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            sts128(reg + ((uint32_t(c) ^ (uint32_t(r) & 7u)) << 4),
                   make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]));
        }
        fence_proxy_async_smem();
        named_bar_sync(2, 128);
        if (r == 0) {
          tma_reduce_add_4d(&tmDQ, sDS, half * 64, 0, t0q, bg);
          tma_reduce_add_4d(&tmDQ, sDS + kBwdRegion, half * 64 + 32, 0, t0q, bg);
          bulk_commit_group();
          bulk_wait_read_all();
        }
        named_bar_sync(2, 128);
      }
      tc_fence_before();
      mbar_arrive(bar(bars->dq_free));
    }
    if (r == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================ 2b. sequence part, d = 128,
// query tiles processed as two 64-row halves
//
// Same algorithm as moda_bwd_seq_kernel, software-pipelined over the two 64-row halves h
// of each query tile so that one half's P/dS math and dQ readout overlap the other
// half's tensor-core products.  TMEM: region A_h = columns [64h, 64h+64) holds S^T_h,
// then P^T_h (bf16 hi/lo), then dQ^T_h; region B_h = [128+64h, 128+64h+64) holds dP^T_h,
// then dS^T_h (hi/lo); dV [256,384), dK [384,512).  dQ^T_h = K^T dS_h^T is an M = 128
// (head-dimension lanes) product, so every tensor-core result keeps the 128-lane layout.
// The dQ warps read dQ^T_h out of TMEM (thread = head-dimension column), release the
// region at once and add the values to the fp32 accumulator with global reductions, a
// warp covering 128 consecutive bytes of one row.  An SM moves about 40 GB/s into L2
// either way (TMA bulk reduce-add or per-thread reductions), so the readout is bound by
// that outbound rate; reductions from registers keep it off the tensor pipe's critical
// path: no shared-memory staging, no wait for the TMA unit before TMEM is released.
// Each tile's row terms (-lse*log2e, -D*scale per row) arrive with its Q in one bulk copy
// from records the depth kernel wrote, so the P/dS warps issue no global loads.
//
// Tensor-core issue order of half h's issuer per tile i (primes: tile i+1; brackets: the
// barrier waited for):
//   [pds_h] dV_h dQ_h dK_h  [qdo'] dP_h'  [dqfree_h] S_h'
// dQ_h comes second so that its readout, which S_h' waits for, starts early.  The two
// issuers share the tensor pipe, so one half's products run while the P/dS warps work on
// the other half, and neither issuer waits behind the other half's barriers.  (So the two
// halves' dV and dK products are summed in whichever order they reach the pipe.)
// warps 0-7 P/dS, 8-11 dQ, 12 TMA, 13 and 14 tcgen05 issuers of halves 0 and 1
constexpr int kSeqHThreads = 480;
constexpr uint32_t kRowTermBytes = 2 * 128 * 4;  // one tile's -lse*log2e and -D records

struct SeqHBars {
  uint64_t kv_full;
  uint64_t qdo_full[2], qdo_empty[2];  // Q, dO and row terms of a tile stage
  uint64_t s_full[2], pds_full[2], dq_full[2], dq_free[2];  // s_full: S and dP landed
  uint64_t kv_done, acc_zero;
  uint32_t tmem_base;
  int abort;
  int lo_tile[2];  // half h of tile i needs its lo passes iff lo_tile[h] == i + 1
};

// The lo halves of P and dS (x - bf16(x)) enter the dV and dK products only for the half
// tiles where some P or |dS| exceeds kLoKeep.  A lo value is at most 2^-8 of its element
// (bf16 keeps 8 significant bits), so every lo value dropped is under 2^-15, and a half
// tile's 64 such terms move a dV or dK entry by far less than the output's own bf16
// rounding.  Large weights (short sequences, the first rows of long ones) keep both passes.
// A warp computes the lo halves of its elements only when one of them is that large, and
// writes zeros otherwise, for the half tiles whose lo passes another warp asked for.
#ifndef MODA_BWD_LO_KEEP
#define MODA_BWD_LO_KEEP 0.0078125f  // 2^-7
#endif
constexpr float kLoKeep = MODA_BWD_LO_KEEP;

// dQ warps of moda_bwd_seq_h_kernel.  Thread = TMEM lane = head-dimension index c of
// dQ^T_h: per half it reads its 64 row values, frees the TMEM region at once and adds
// the values to the fp32 accumulator with global reductions (a warp covers 32
// consecutive columns of one row: 128 bytes).  Half row r is tile row R = 64h + r, i.e.
// token R / G and head R % G.  GT = G for a power of two up to 16, so that each row's
// offset from its head's base pointer is a compile-time constant; GT = 0 handles any G.
template <int GT>
__device__ __forceinline__ void dq_readout(const SeqArgs& a, SeqHBars* bars, uint32_t tmem,
                                           uint32_t lane_base, int c, int bg, int first_qt,
                                           int ntiles) {
  constexpr int D = 128;
  volatile int* abort_flag = &bars->abort;
  const long long hs = (long long)a.T * D;
  for (int i = 0; i < ntiles; ++i) {
    const int t0q = (first_qt + i) * a.TQ;
    const int ntok = min(a.TQ, a.T - t0q);  // valid tokens of this tile
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      const uint32_t tA = tmem + uint32_t(64 * h);  // region A_h
      mbar_wait(smem_u32(&bars->dq_full[h]), i & 1, abort_flag);
      tc_fence_after();
      uint32_t o[64];
      tmem_ld32(tA + lane_base, o);
      tmem_ld32(tA + lane_base + 32, o + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->dq_free[h]));
      if constexpr (GT > 0) {
        const int tok0 = (64 * h) / GT;
        const int nv = ntok - tok0;
        float* const base = a.dqacc + ((long long)bg * GT * a.T + t0q + tok0) * D + c;
        // rows in order (heads cycling fastest), in blocks of up to four heads so that at
        // most four base pointers are live; issuing the rows in order measured faster
        // than head by head
        constexpr int HB = GT < 4 ? GT : 4;
#pragma unroll
        for (int hb = 0; hb < GT / HB; ++hb) {
          float* ph[HB];
#pragma unroll
          for (int j = 0; j < HB; ++j) ph[j] = base + (hb * HB + j) * hs;
#pragma unroll
          for (int tk = 0; tk < 64 / GT; ++tk)
#pragma unroll
            for (int j = 0; j < HB; ++j)
              if (tk < nv) red_add_f32(ph[j] + tk * D, __uint_as_float(o[tk * GT + hb * HB + j]));
        }
      } else {
        float* const base = a.dqacc + ((long long)bg * a.G * a.T + t0q) * D + c;
#pragma unroll
        for (int r = 0; r < 64; ++r) {
          const int R = 64 * h + r;
          const int tok = R / a.G;
          if (tok < ntok)
            red_add_f32(base + (R - tok * a.G) * hs + tok * D, __uint_as_float(o[r]));
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kSeqHThreads, 1)
    moda_bwd_seq_h_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmDO,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const SeqArgs a) {
  constexpr int D = 128;
  using Cfg = SeqCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicOr(&g_error_word, kErrInternal);
    return;
  }
  const uint32_t s0 = smem_u32(smem);
  const uint32_t sK = s0 + Cfg::kOffK, sV = s0 + Cfg::kOffV, sDS = s0 + Cfg::kOffDS;
  auto sQ = [&](int st) { return s0 + Cfg::kOffQ + uint32_t(st) * Cfg::kTile; };
  auto sDO = [&](int st) { return s0 + Cfg::kOffDO + uint32_t(st) * Cfg::kTile; };
  auto sLD = [&](int st) { return s0 + Cfg::kOffLD + uint32_t(st) * kRowTermBytes; };
  const float* ld_s = reinterpret_cast<const float*>(smem + Cfg::kOffLD);
  SeqHBars* bars = reinterpret_cast<SeqHBars*>(smem + Cfg::kOffBar);
  volatile int* abort_flag = &bars->abort;
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };

  const int warp = threadIdx.x >> 5;
  const int bg = blockIdx.x % a.BG;
  const int kb = blockIdx.x / a.BG;
  const int key0 = kb * 128;
  const int first_qt = a.causal ? key0 / a.TQ : 0;
  const int ntiles = a.nqt - first_qt;

  if (threadIdx.x == 0) {
    mbar_init(bar(bars->kv_full), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(bars->qdo_full[i]), 1);
      mbar_init(bar(bars->qdo_empty[i]), 2);  // one commit from each issuer
      mbar_init(bar(bars->s_full[i]), 1);
      mbar_init(bar(bars->pds_full[i]), 256);
      mbar_init(bar(bars->dq_full[i]), 1);
      mbar_init(bar(bars->dq_free[i]), 128);
    }
    mbar_init(bar(bars->kv_done), 2);
    mbar_init(bar(bars->acc_zero), 256);
    bars->abort = 0;
    bars->lo_tile[0] = bars->lo_tile[1] = 0;
    fence_barrier_init();
  }
  // Q/dO rows past TQ*G (G not dividing 128) never receive TMA data: zero them once.
  if (threadIdx.x < 128 && threadIdx.x >= a.TQ * a.G) {
    for (int st = 0; st < 2; ++st)
      for (int rg = 0; rg < Cfg::kRegions; ++rg) {
        uint4* rq = reinterpret_cast<uint4*>(smem + Cfg::kOffQ + st * Cfg::kTile +
                                             rg * kBwdRegion + threadIdx.x * 128);
        uint4* rd = reinterpret_cast<uint4*>(smem + Cfg::kOffDO + st * Cfg::kTile +
                                             rg * kBwdRegion + threadIdx.x * 128);
        for (int c = 0; c < 8; ++c) rq[c] = rd[c] = make_uint4(0, 0, 0, 0);
      }
    fence_proxy_async_smem();
  }
  volatile int* lo_tile = bars->lo_tile;
  if (warp == 13) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  auto tA = [&](int h) { return tmem + uint32_t(64 * h); };
  auto tB = [&](int h) { return tmem + uint32_t(128 + 64 * h); };
  const uint32_t tDV = tmem + 256, tDK = tmem + 384;

  if (warp == 12) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmDO);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(bar(bars->kv_full), 2 * Cfg::kTile);
      for (int rg = 0; rg < Cfg::kRegions; ++rg) {
        tma_load_3d(sK + rg * kBwdRegion, &tmK, bar(bars->kv_full), rg * 64, key0, bg);
        tma_load_3d(sV + rg * kBwdRegion, &tmV, bar(bars->kv_full), rg * 64, key0, bg);
      }
      const uint32_t qbytes = Cfg::kRegions * 128 * a.G * a.TQ;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i & 1;
        const int t0 = (first_qt + i) * a.TQ;
        // qdo_empty also means every P/dS warp is done with tile i-2's row terms
        if (i >= 2) mbar_wait(bar(bars->qdo_empty[st]), ((i >> 1) - 1) & 1, abort_flag);
        const uint32_t full = bar(bars->qdo_full[st]);
        mbar_expect_tx(full, 2 * qbytes + kRowTermBytes);
        bulk_load(sLD(st), a.rt + ((long long)bg * a.nqt + first_qt + i) * 256, kRowTermBytes,
                  full);
        for (int rg = 0; rg < Cfg::kRegions; ++rg) {
          tma_load_4d(sQ(st) + rg * kBwdRegion, &tmQ, full, rg * 64, 0, t0, bg);
          tma_load_4d(sDO(st) + rg * kBwdRegion, &tmDO, full, rg * 64, 0, t0, bg);
        }
      }
    }
    __syncwarp();
  } else if (warp == 13 || warp == 14) {
    // ------------------------------------------------------------ tcgen05 issuers
    // One issuer per 64-row half, so that neither half's products wait behind a barrier
    // of the other half; both feed the SM's one tensor pipe.  dV and dK accumulate the
    // products of both issuers: the P/dS warps zero them first, and every product adds.
    const int h = warp - 13;
    if (elect_one()) {
      constexpr uint32_t idesc_t = make_idesc_bf16(128, 64, 0, 0);  // S^T_h, dP^T_h
      constexpr uint32_t idesc_g = make_idesc_bf16(128, D, 0, 1);   // dV, dK (A in TMEM)
      constexpr uint32_t idesc_q = make_idesc_bf16(128, 64, 1, 1);  // dQ^T_h = K^T dS_h^T
      mbar_wait(bar(bars->kv_full), 0, abort_flag);
      // S^T_h(i) = K Q_h(i)^T, dP^T_h(i) = V dO_h(i)^T : B = the half's 64 rows, K-major
      auto wait_qdo = [&](int i) {
        mbar_wait(bar(bars->qdo_full[i & 1]), (i >> 1) & 1, abort_flag);
      };
      // (qdo_full of tile i waited for beforehand)
      auto issue_s = [&](int i, int h) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks / 4) * kBwdRegion + (ks % 4) * 32;
          mma_ss(tA(h), make_sdesc_sw128(sK + off, 16, 1024),
                 make_sdesc_sw128(sQ(i & 1) + off + 8192 * h, 16, 1024), idesc_t,
                 ks > 0 ? 1u : 0u);
        }
        tc_commit(bar(bars->s_full[h]));
      };
      auto issue_dp = [&](int i, int h) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks / 4) * kBwdRegion + (ks % 4) * 32;
          mma_ss(tB(h), make_sdesc_sw128(sV + off, 16, 1024),
                 make_sdesc_sw128(sDO(i & 1) + off + 8192 * h, 16, 1024), idesc_t,
                 ks > 0 ? 1u : 0u);
        }
        // no commit of its own: the S product's commit, always issued later by this
        // thread, tracks these products too
      };
      // dV += P_h^T dO_h, dK += dS_h^T Q_h (hi then lo; K-step ks covers the half's rows
      // 16ks..16ks+15: packed columns 32(ks/2) + 8(ks%2) of the region, lo +16), then
      // dQ^T_h = K^T dS_h^T into region A_h, after dV has read P^T_h from it.
      auto issue_grads = [&](int i, int h) {
        mbar_wait(bar(bars->pds_full[h]), i & 1, abort_flag);
        tc_fence_after();
        // dV (reads P^T_h), then dQ^T_h over P^T_h, then dK (reads dS^T_h from B_h): the
        // dQ readout, which the next S product waits for, starts as early as it can
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_ts(tDV, tA(h) + (ks >> 1) * 32 + (ks & 1) * 8,
                 make_sdesc_sw128(sDO(i & 1) + (4 * h + ks) * 2048, kBwdRegion, 1024), idesc_g,
                 1u);
        // the lo products, if the P/dS warps marked the half (before arriving on pds_full);
        // the flag is read only now, so that its latency overlaps the products above
        const bool lo = lo_tile[h] == i + 1;
        if (lo) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ts(tDV, tA(h) + (ks >> 1) * 32 + (ks & 1) * 8 + 16,
                   make_sdesc_sw128(sDO(i & 1) + (4 * h + ks) * 2048, kBwdRegion, 1024),
                   idesc_g, 1u);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tA(h), make_sdesc_sw128(sK + ks * 2048, kBwdRegion, 1024),
                 make_sdesc_sw128(sDS + h * kBwdRegion + ks * 2048, kBwdRegion, 1024), idesc_q,
                 ks > 0 ? 1u : 0u);
        tc_commit(bar(bars->dq_full[h]));
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t col = (ks >> 1) * 32 + (ks & 1) * 8;
          const uint64_t bq =
              make_sdesc_sw128(sQ(i & 1) + (4 * h + ks) * 2048, kBwdRegion, 1024);
          mma_ts(tDK, tB(h) + col, bq, idesc_g, 1u);
          if (lo) mma_ts(tDK, tB(h) + col + 16, bq, idesc_g, 1u);
        }
      };
      // dP before S in every tile: the commit of S then also covers dP, so the P/dS warps
      // wait for S alone
      wait_qdo(0);
      issue_dp(0, h);
      issue_s(0, h);
      mbar_wait(bar(bars->acc_zero), 0, abort_flag);
      tc_fence_after();
      for (int i = 0; i < ntiles; ++i) {
        // one early test for the next tile's Q and dO, while this half's P/dS is still
        // being computed: when they have landed, dP' below needs no wait of its own
        const bool qdo_seen =
            i + 1 < ntiles &&
            mbar_try_wait(bar(bars->qdo_full[(i + 1) & 1]), ((i + 1) >> 1) & 1);
        issue_grads(i, h);
        tc_commit(bar(bars->qdo_empty[i & 1]));  // Q(i), dO(i): this half's products read
        if (i + 1 < ntiles) {
          if (!qdo_seen) wait_qdo(i + 1);
          issue_dp(i + 1, h);  // region B_h: dK has read dS^T_h
          mbar_wait(bar(bars->dq_free[h]), i & 1, abort_flag);
          issue_s(i + 1, h);
        }
      }
      tc_commit(bar(bars->kv_done));
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ P / dS warps
    // Two warps per TMEM sub-partition: warp w owns key lanes 32(w%4)..32(w%4)+31 and, in
    // each 64-row half, the 32-row chunk g = w/4.
    const int g = warp >> 2;
    const int kt = threadIdx.x & 127;  // TMEM lane = key key0 + kt
    const int key = key0 + kt;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const float2 sl2 = make_float2(a.scale_log2, a.scale_log2);
    const float2 sc2 = make_float2(a.scale, a.scale);
    const float2 neg1 = make_float2(-1.f, -1.f);
    {
      // this lane's row of the dV (group 0) or dK (group 1) accumulator starts at zero
      const uint32_t zero8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      const uint32_t dst = (g ? tDK : tDV) + lane_base;
#pragma unroll
      for (int cc = 0; cc < D / 8; ++cc) tmem_st8(dst + 8 * cc, zero8);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(bars->acc_zero));
    }
    for (int i = 0; i < ntiles; ++i) {
      const int qt = first_qt + i;
      const int b = i & 1;
      // The tile's row terms came with its Q and dO: the issuer saw them land (qdo_full)
      // before it issued S, and the s_full wait below orders them before the reads.
      int r_min = 0;
      if (key >= a.T)
        r_min = 1 << 30;
      else if (a.causal)
        r_min = a.G * (key - qt * a.TQ);
      const float* nlse2 = ld_s + b * 256;       // -lse * log2e per tile row
      const float* ndr = ld_s + b * 256 + 128;   // -D * scale per tile row
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        // S's commit came after dP's from the same issuer, so it covers both products
        mbar_wait(bar(bars->s_full[h]), i & 1, abort_flag);
        tc_fence_after();
        const int c = 2 * h + g;  // 32-row chunk of the tile
        // the packed results overwrite these columns: load all 32 before storing any
        uint32_t s[32], dp[32];
        tmem_ld32(tA(h) + lane_base + g * 32, s);
        tmem_ld32(tB(h) + lane_base + g * 32, dp);
        // row terms of one 16-row sub-chunk, read while the TMEM loads are in flight (the
        // TMEM wait and the stores below order shared memory, so loads placed after them
        // would wait for them)
        float4 nlk[4], ndk[4];
        auto load_rt = [&](int k) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int r4 = c * 32 + 16 * k + 4 * q4;
            nlk[q4] = *reinterpret_cast<const float4*>(nlse2 + r4);
            ndk[q4] = *reinterpret_cast<const float4*>(ndr + r4);
          }
        };
        load_rt(0);
        tmem_wait_ld();
        const bool masked = r_min > c * 32;
        // dS for the dQ^T product: region h, this key's row, rows 32g..32g+31 of the half
        const uint32_t reg = sDS + h * kBwdRegion + uint32_t(kt) * 128;
        const uint32_t tP = tA(h) + lane_base + g * 32, tS = tB(h) + lane_base + g * 32;
        // One pass over this thread's 32 elements: P = 2^(s*scale*log2e - lse*log2e) and
        // dS = P * scale*(dP - D) (both row terms stored negated, D pre-scaled).  The first
        // pass stores the bf16 P^T / dS^T words (hi, chunk columns 8k..) and returns the
        // largest P or |dS|; kLo passes store what the rounding dropped (lo, 16 columns
        // further).
        auto pass = [&](auto lo_c) {
          constexpr bool kLo = decltype(lo_c)::value;
          float mx = 0.f;
          if constexpr (kLo) load_rt(0);
#pragma unroll
          for (int k = 0; k < 2; ++k) {  // 16-row sub-chunks
            uint32_t hp[8], hd[8], lp[8], ld[8];
#pragma unroll
            for (int e4 = 0; e4 < 16; e4 += 4) {
              const float4 nl = nlk[e4 >> 2], nd = ndk[e4 >> 2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int e = 16 * k + e4 + 2 * u, w = (e4 >> 1) + u;
                const float2 arg = ffma2(
                    make_float2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), sl2,
                    u ? make_float2(nl.z, nl.w) : make_float2(nl.x, nl.y));
                const float P0 = ex2(arg.x), P1 = ex2(arg.y);
                const float2 dd = ffma2(
                    make_float2(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])), sc2,
                    u ? make_float2(nd.z, nd.w) : make_float2(nd.x, nd.y));
                const float2 dS = fmul2(make_float2(P0, P1), dd);
                const uint32_t ph = pack_bf16x2(P0, P1), dh = pack_bf16x2(dS.x, dS.y);
                if constexpr (kLo) {
                  const float2 plo =
                      ffma2(make_float2(bf16lo(ph), bf16hi(ph)), neg1, make_float2(P0, P1));
                  const float2 dlo = ffma2(make_float2(bf16lo(dh), bf16hi(dh)), neg1, dS);
                  lp[w] = pack_bf16x2(plo.x, plo.y);
                  ld[w] = pack_bf16x2(dlo.x, dlo.y);
                } else {
                  hp[w] = ph;
                  hd[w] = dh;
                  mx = fmax3(mx, P0, P1);
                  mx = fmax3(mx, fabsf(dS.x), fabsf(dS.y));
                }
              }
            }
            if (k == 0) load_rt(1);  // before the stores, which order shared memory
            if constexpr (kLo) {
              tmem_st8(tP + 16 + 8 * k, lp);
              tmem_st8(tS + 16 + 8 * k, ld);
            } else {
              tmem_st8(tP + 8 * k, hp);
              tmem_st8(tS + 8 * k, hd);
#pragma unroll
              for (int qd = 0; qd < 2; ++qd) {
                const uint32_t chunk = g * 4 + 2 * k + qd;
                sts128(reg + ((chunk ^ (uint32_t(kt) & 7u)) << 4),
                       make_uint4(hd[qd * 4], hd[qd * 4 + 1], hd[qd * 4 + 2], hd[qd * 4 + 3]));
              }
            }
          }
          return mx;
        };
        using kNo = std::integral_constant<bool, false>;
        using kYes = std::integral_constant<bool, true>;
        // A masked score (causal, or a key past the end) becomes -inf before the pass, so
        // its P and dS are 0, in the few warps that hold a masked row (r_min <= 32c for a
        // thread without one); the pass itself has one form.
        if (__any_sync(0xffffffffu, masked)) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e < r_min) s[e] = __float_as_uint(-INFINITY);
        }
        const float mx = pass(kNo{});
        if (__any_sync(0xffffffffu, mx > kLoKeep)) {
          pass(kYes{});
          // mark the half for its lo passes (ordered before this lane's arrival below)
          if ((threadIdx.x & 31) == 0) lo_tile[h] = i + 1;
        } else {
          // zeros: the lo passes, if another warp's rows need them, add nothing for these
          const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            tmem_st8(tP + 16 + 8 * k, z);
            tmem_st8(tS + 16 + 8 * k, z);
          }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(bars->pds_full[h]));
      }
    }
    // epilogue: group 0 writes this key's dV row, group 1 its dK row
    mbar_wait(bar(bars->kv_done), 0, abort_flag);
    tc_fence_after();
    const bool kvalid = key < a.T;
    const long long koff = ((long long)bg * a.T + (kvalid ? key : 0)) * D;
    {
      const uint32_t tsrc = (g ? tDK : tDV) + lane_base;
      __nv_bfloat16* dst = (g ? a.dk : a.dv) + koff;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tsrc + cc * 32, o);
        tmem_wait_ld();
        if (kvalid) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(o[v * 8 + e]);
            d4[v] = pack8(f, 1.f);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ dQ warps 8-11
    // Thread = TMEM lane = head-dimension index c of dQ^T_h: it reads its 64 row values,
    // frees the TMEM region, and adds them to the fp32 accumulator with global
    // reductions (a warp covers 32 consecutive columns of one row: 128 bytes).
    const int c = threadIdx.x - 256;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    switch (a.G) {
      case 1: dq_readout<1>(a, bars, tmem, lane_base, c, bg, first_qt, ntiles); break;
      case 2: dq_readout<2>(a, bars, tmem, lane_base, c, bg, first_qt, ntiles); break;
      case 4: dq_readout<4>(a, bars, tmem, lane_base, c, bg, first_qt, ntiles); break;
      case 8: dq_readout<8>(a, bars, tmem, lane_base, c, bg, first_qt, ntiles); break;
      case 16: dq_readout<16>(a, bars, tmem, lane_base, c, bg, first_qt, ntiles); break;
      default: dq_readout<0>(a, bars, tmem, lane_base, c, bg, first_qt, ntiles); break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================ 3. dq convert
__global__ void __launch_bounds__(256) moda_dq_convert_kernel(const float* __restrict__ acc,
                                                              __nv_bfloat16* __restrict__ dq,
                                                              long long n8) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 x = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 y = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    const float f[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
    reinterpret_cast<uint4*>(dq)[i] = pack8(f, 1.f);
  }
}

// ============================================================ host side
bool make_map_b(EncodeTiledFn encode, CUtensorMap* map, const void* base, int rank,
                const cuuint64_t* dims, const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int D, int GM, bool kRT>
cudaError_t launch_depth(const BwdDepthArgs& args, cudaStream_t stream, const char** why) {
  const int tpb = kDepthThreads / (D / 8);
  BwdDepthArgs a = args;
  // depth-only attention with q and dO in registers: stage the first pass's (P, <dO, vd>)
  // pairs when a CTA's tokens' pairs fit in the ring's second half
  a.staged = (!kRT && GM <= 4 && a.exact_rows && a.acc_mode == 0 &&
              (long long)tpb * a.L * GM * 8 <= kDepthStageBytes)
                 ? 1
                 : 0;
  // q/dO slots (not needed when they live in registers) + the per-thread cp.async ring
  const size_t smem = (GM <= 4 ? 0 : size_t(tpb) * 2 * a.G * D * 2) + kDepthRingBytes;
  cudaError_t e = cudaFuncSetAttribute(moda_bwd_depth_kernel<D, GM, kRT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) {
    *why = "cudaFuncSetAttribute(depth backward) failed";
    return e;
  }
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, moda_bwd_depth_kernel<D, GM, kRT>,
                                                kDepthThreads, smem);
  if (per_sm < 1) per_sm = 1;
  const long long need = (a.ntok + tpb - 1) / tpb;
  const long long cap = (long long)sm_count() * per_sm;
  const unsigned grid = unsigned(need < cap ? need : cap);
  moda_bwd_depth_kernel<D, GM, kRT><<<grid, kDepthThreads, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) *why = "depth backward launch failed";
  return e;
}

// Byte offsets of the backward's workspace regions: the fp32 dq accumulator [B][Hq][T][d]
// at 0, the head-major row terms D [B][Hq][T] (d = 64), the tiled row-term records
// [B*Hkv][nqt][2][128] (d = 128), then the fp32 dkd/dvd accumulators of groups above
// kDepthMaxG heads.
struct BwdLayout {
  size_t drow, rt, acc;
};
inline BwdLayout bwd_layout(const Problem& p) {
  const size_t rows = size_t(p.B) * p.Hq * p.T;
  BwdLayout l;
  l.drow = rows * p.d * 4;
  l.rt = (l.drow + rows * 4 + 255) & ~size_t(255);
  const size_t rt_bytes =
      p.d == 128 ? size_t(p.B) * p.Hkv * tile_geom(p).nqt * kRowTermBytes : 0;
  l.acc = l.rt + rt_bytes;
  return l;
}

template <int D>
cudaError_t launch_backward_d(const Problem& p, const void* q, const void* k, const void* v,
                              const void* kd, const void* vd, const void* out,
                              const float* lse, const void* dout, void* dq, void* dk,
                              void* dv, void* dkd, void* dvd, void* workspace,
                              unsigned stages, EncodeTiledFn encode, cudaStream_t stream,
                              const char** why) {
  const TileGeom tg = tile_geom(p);
  const long long rows = (long long)p.B * p.Hq * p.T;
  const BwdLayout lay = bwd_layout(p);
  uint8_t* const ws = static_cast<uint8_t*>(workspace);
  float* dqacc = reinterpret_cast<float*>(ws);
  float* drow = reinterpret_cast<float*>(ws + lay.drow);
  float* rt = reinterpret_cast<float*>(ws + lay.rt);

  // 1. depth part, row terms, dq accumulator initialisation
  BwdDepthArgs da;
  da.q = static_cast<const __nv_bfloat16*>(q);
  da.out = static_cast<const __nv_bfloat16*>(out);
  da.dout = static_cast<const __nv_bfloat16*>(dout);
  da.kd = static_cast<const __nv_bfloat16*>(kd);
  da.vd = static_cast<const __nv_bfloat16*>(vd);
  da.lse = lse;
  da.dkd = static_cast<__nv_bfloat16*>(dkd);
  da.dvd = static_cast<__nv_bfloat16*>(dvd);
  da.dqacc = dqacc;
  // the d = 64 sequence kernel reads head-major row terms, the d = 128 one tiled records;
  // depth-only attention has no sequence part
  da.drow = (D == 64 && !p.depth_only) ? drow : nullptr;
  da.rt = (D == 128 && !p.depth_only) ? rt : nullptr;
  da.TQ = tg.TQ;
  da.nqt = tg.nqt;
  da.ntok = (long long)p.B * p.Hkv * p.T;
  da.T = p.T;
  da.L = p.L;
  da.G = p.G;
  da.head0 = 0;
  da.Gfull = p.G;
  da.acc_mode = 0;
  da.dkd_acc = da.dvd_acc = nullptr;
  da.exact_rows = p.depth_only;
  da.staged = 0;  // (decided per launch in launch_depth)
  da.scale = p.scale;
  da.scale_log2 = p.scale * kLog2eBwd;
  cudaError_t e = cudaSuccess;
  if (stages & kStageDepth) {
    auto launch = [&]() {
      constexpr bool kRT = D == 128;  // (depth-only attention: rt is null, below)
      if (da.rt == nullptr) {
        if (da.G <= 1) return launch_depth<D, 1, false>(da, stream, why);
        if (da.G <= 2) return launch_depth<D, 2, false>(da, stream, why);
        if (da.G <= 4) return launch_depth<D, 4, false>(da, stream, why);
        if (da.G <= 8) return launch_depth<D, 8, false>(da, stream, why);
        return launch_depth<D, 16, false>(da, stream, why);
      }
      if (da.G <= 1) return launch_depth<D, 1, kRT>(da, stream, why);
      if (da.G <= 2) return launch_depth<D, 2, kRT>(da, stream, why);
      if (da.G <= 4) return launch_depth<D, 4, kRT>(da, stream, why);
      if (da.G <= 8) return launch_depth<D, 8, kRT>(da, stream, why);
      return launch_depth<D, 16, kRT>(da, stream, why);
    };
    if (p.G <= kDepthMaxG) {
      e = launch();
    } else {
      // one launch per chunk of kDepthMaxG heads; dkd/dvd summed in fp32 in the workspace
      // after the dq accumulator and the row terms
      const size_t nd = size_t(p.B) * p.Hkv * p.T * size_t(p.L) * D;
      da.dkd_acc = reinterpret_cast<float*>(ws + lay.acc);
      da.dvd_acc = da.dkd_acc + nd;
      const int nchunk = (p.G + kDepthMaxG - 1) / kDepthMaxG;
      for (int c = 0; c < nchunk && e == cudaSuccess; ++c) {
        da.head0 = c * kDepthMaxG;
        da.G = min(kDepthMaxG, p.G - da.head0);
        da.acc_mode = p.L == 0 ? 0 : (c == 0 ? 1 : (c == nchunk - 1 ? 3 : 2));
        e = launch();
      }
    }
    if (e != cudaSuccess) return e;
  }
  // 2. sequence part (none for depth-only attention)
  if (stages & kStageSeq) {
    const cuuint64_t E = 2;
    const cuuint64_t BG = cuuint64_t(p.B) * p.Hkv;
    CUtensorMap mQ, mDO, mK, mV;
    {
      const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(p.G), cuuint64_t(p.T), BG};
      const cuuint64_t str[3] = {cuuint64_t(p.T) * D * E, cuuint64_t(D) * E,
                                 cuuint64_t(p.G) * p.T * D * E};
      const cuuint32_t box[4] = {64, cuuint32_t(p.G), cuuint32_t(tg.TQ), 1};
      if (!make_map_b(encode, &mQ, q, 4, dims, str, box) ||
          !make_map_b(encode, &mDO, dout, 4, dims, str, box)) {
        *why = "cuTensorMapEncodeTiled failed for q/dout";
        return cudaErrorInvalidValue;
      }
    }
    {
      const cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(p.T), BG};
      const cuuint64_t str[2] = {cuuint64_t(D) * E, cuuint64_t(p.T) * D * E};
      const cuuint32_t box[3] = {64, 128, 1};
      if (!make_map_b(encode, &mK, k, 3, dims, str, box) ||
          !make_map_b(encode, &mV, v, 3, dims, str, box)) {
        *why = "cuTensorMapEncodeTiled failed for k/v";
        return cudaErrorInvalidValue;
      }
    }
    SeqArgs sa;
    sa.dk = static_cast<__nv_bfloat16*>(dk);
    sa.dv = static_cast<__nv_bfloat16*>(dv);
    sa.dqacc = dqacc;
    sa.lse = lse;
    sa.drow = drow;
    sa.rt = rt;
    sa.Hkv = p.Hkv;
    sa.T = p.T;
    sa.G = p.G;
    sa.TQ = tg.TQ;
    sa.nqt = tg.nqt;
    sa.BG = int(BG);
    sa.causal = p.causal;
    sa.scale = p.scale;
    sa.scale_log2 = p.scale * kLog2eBwd;
    const int nkb = (p.T + 127) / 128;
    if constexpr (D == 128) {
      e = cudaFuncSetAttribute(moda_bwd_seq_h_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SeqCfg<128>::kSmemBytes);
      if (e != cudaSuccess) {
        *why = "cudaFuncSetAttribute(sequence backward, halves) failed";
        return e;
      }
      moda_bwd_seq_h_kernel<<<unsigned(BG) * nkb, kSeqHThreads, SeqCfg<128>::kSmemBytes,
                              stream>>>(mQ, mDO, mK, mV, sa);
    } else {
      CUtensorMap mDQ;
      // fp32 dq accumulator viewed like q: [bg][t][head-in-group][c]; a box is 32 columns
      // (128 bytes) of one tile's rows (token, head), 128B-swizzled.
      const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(p.G), cuuint64_t(p.T), BG};
      const cuuint64_t str[3] = {cuuint64_t(p.T) * D * 4, cuuint64_t(D) * 4,
                                 cuuint64_t(p.G) * p.T * D * 4};
      const cuuint32_t box[4] = {32, cuuint32_t(p.G), cuuint32_t(tg.TQ), 1};
      cuuint32_t estr[5] = {1, 1, 1, 1, 1};
      if (encode(&mDQ, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dqacc, dims, str, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        *why = "cuTensorMapEncodeTiled failed for the dq accumulator";
        return cudaErrorInvalidValue;
      }
      e = cudaFuncSetAttribute(moda_bwd_seq_kernel<D>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SeqCfg<D>::kSmemBytes);
      if (e != cudaSuccess) {
        *why = "cudaFuncSetAttribute(sequence backward) failed";
        return e;
      }
      moda_bwd_seq_kernel<D><<<unsigned(BG) * nkb, kSeqThreads, SeqCfg<D>::kSmemBytes, stream>>>(
          mQ, mDO, mK, mV, mDQ, sa);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) {
      *why = "sequence backward launch failed";
      return e;
    }
  }

  // 3. dq (bf16)
  if (!(stages & kStageConvert)) return cudaSuccess;
  const long long n8 = rows * D / 8;
  long long blocks = (n8 + 255) / 256;
  if (blocks > 8LL * sm_count()) blocks = 8LL * sm_count();
  moda_dq_convert_kernel<<<unsigned(blocks), 256, 0, stream>>>(
      dqacc, static_cast<__nv_bfloat16*>(dq), n8);
  e = cudaGetLastError();
  if (e != cudaSuccess) *why = "dq convert launch failed";
  return e;
}

}  // namespace

size_t backward_workspace_bytes(const Problem& p) {
  const BwdLayout lay = bwd_layout(p);
  size_t bytes = lay.acc;
  // groups above kDepthMaxG heads: fp32 dkd and dvd accumulators for the chunked depth part
  if (p.G > kDepthMaxG) bytes += 2 * size_t(p.B) * p.Hkv * p.T * size_t(p.L) * p.d * 4;
  return bytes;
}

cudaError_t launch_backward(const Problem& p, const void* q, const void* k, const void* v,
                            const void* kd, const void* vd, const void* out, const float* lse,
                            const void* dout, void* dq, void* dk, void* dv, void* dkd,
                            void* dvd, void* workspace, unsigned stages,
                            EncodeTiledFn encode, cudaStream_t stream, const char** why) {
  if (p.d == 128)
    return launch_backward_d<128>(p, q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd,
                                  workspace, stages, encode, stream, why);
  return launch_backward_d<64>(p, q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd,
                               workspace, stages, encode, stream, why);
}

}  // namespace moda
