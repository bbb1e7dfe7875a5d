// moda_internal.h -- shared declarations between the host entry points (moda_api.cu)
// and the kernel launchers.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moda {

// Geometry of one forward/backward problem after validation.
struct Problem {
  int B, Hq, Hkv, T, L, d, G;
  int causal;
  float scale;
  int depth_only = 0;  // 1: no sequence keys (depth-only attention); k, v unused
};

// Tile geometry shared by the kernels: a query tile holds 128 (token, head) rows, TQ
// tokens x G heads of one KV group, token-major (row r = token*G + head); depth chunks
// hold JC depth entries of the tile's TQ tokens.
struct TileGeom {
  int TQ;   // tokens per query tile = 128 / G (floor)
  int JC;   // depth entries per depth chunk = min(8, 128 / TQ)
  int nqt;  // query tiles per (b, kv head) = ceil(T / TQ)
};

inline TileGeom tile_geom(const Problem& p) {
  TileGeom t;
  t.TQ = 128 / p.G;
  t.JC = 128 / t.TQ;
  if (t.JC > 8) t.JC = 8;
  t.nqt = (p.T + t.TQ - 1) / t.TQ;
  return t;
}

// Tensor-map encoder obtained from the driver at run time (no link-time libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

// Forward depth paths: the CUDA-core fold (each tile's depth rows folded into the softmax
// state on CUDA cores before its sequence blocks) or dense depth blocks (the depth rows
// run through the tensor-core pipeline as extra masked 128-key blocks; needs G | 128).
constexpr int kDepthPathAuto = 0, kDepthPathFold = 1, kDepthPathDense = 2;
// The automatic choice takes dense depth blocks from this many depth entries up (measured
// on B200: as fast or faster than the fold from L = 24 to 128, and at L = 32, 64K tokens).
constexpr int kDenseDepthMinL = 1;
bool dense_depth_supported(const Problem& p);
bool dense_depth_default(const Problem& p);

// Forward launcher: returns a CUDA error code (cudaSuccess when enqueued).
// Test only: y[i] = the forward's FMA-pipe 2^x (exp2_fma2) of x[i], i < n (device arrays).
cudaError_t launch_test_exp2_fma(const float* x, float* y, int n, cudaStream_t stream);

cudaError_t launch_forward(const Problem& p, const void* q, const void* k, const void* v,
                           const void* kd, const void* vd, void* out, float* lse,
                           int depth_path, EncodeTiledFn encode, cudaStream_t stream,
                           const char** why);

cudaError_t launch_backward(const Problem& p, const void* q, const void* k, const void* v,
                            const void* kd, const void* vd, const void* out,
                            const float* lse, const void* dout, void* dq, void* dk,
                            void* dv, void* dkd, void* dvd, void* workspace,
                            unsigned stages, EncodeTiledFn encode, cudaStream_t stream,
                            const char** why);

// Single-token decode: the sequence is split into ranges of 128-key blocks, one CTA per
// (batch, KV head, range); `T` of the Problem is the cache length S.
struct DecodeSplit {
  int nsplit, blocks_per_split;
};
DecodeSplit decode_split(const Problem& p);
size_t decode_workspace_bytes(const Problem& p);
cudaError_t launch_decode(const Problem& p, const void* q, const void* k, const void* v,
                          const void* kd, const void* vd, void* out, float* lse,
                          void* workspace, EncodeTiledFn encode, cudaStream_t stream,
                          const char** why);

// Fused depth-stream write: K|V = X W^T for B*T tokens, stored into slot `slot` of the
// [B, Hkv, T, L, d] depth caches.
struct KvWriteProblem {
  int B, T, hidden, Hkv, d, L, slot;
};
cudaError_t launch_kvwrite(const KvWriteProblem& p, const void* x, const void* w, void* kd,
                           void* vd, EncodeTiledFn encode, cudaStream_t stream,
                           const char** why);

// Backward stages (bit mask): 1 row terms + depth part + dq accumulator initialisation,
// 2 sequence part (adds to the dq accumulator), 4 dq conversion to bf16.
constexpr unsigned kStageDepth = 1u, kStageSeq = 2u, kStageConvert = 4u, kStagesAll = 7u;

size_t backward_workspace_bytes(const Problem& p);

}  // namespace moda
