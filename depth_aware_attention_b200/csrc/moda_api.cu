// moda_api.cu -- the extern "C" entry points declared in include/moda.h.
//
// Host side only: argument validation (before any launch), device capability check,
// the tensor-map encoder obtained from the driver at run time, the per-device kernel
// error word, and status/message reporting.  All arithmetic runs in the kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "../../include/moda.h"
#include "moda_internal.h"
#include "sm100.cuh"

namespace {

thread_local char g_msg[512] = "";

moda_status_t fail(moda_status_t s, const char* fmt, const char* detail = nullptr) {
  if (detail)
    snprintf(g_msg, sizeof(g_msg), fmt, detail);
  else
    snprintf(g_msg, sizeof(g_msg), "%s", fmt);
  return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte ranges [p, p+n) and [q, q+m) overlap?
bool overlaps(const void* p, size_t n, const void* q, size_t m) {
  if (!p || !q || n == 0 || m == 0) return false;
  const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
  return a < b + m && b < a + n;
}

moda_status_t check_sizes(int B, int Hq, int Hkv, int T, int L, int d) {
  if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || L < 0)
    return fail(MODA_ERR_INVALID_ARGUMENT, "sizes must satisfy B,Hq,Hkv,T >= 1 and L >= 0");
  if (Hq % Hkv != 0) return fail(MODA_ERR_INVALID_ARGUMENT, "Hq must be a multiple of Hkv");
  if (d != 64 && d != 128) return fail(MODA_ERR_UNSUPPORTED, "head size d must be 64 or 128");
  // Groups above 64 are refused: a query tile holds 128 / G tokens, and the parity tests
  // cover groups up to 64.
  if (Hq / Hkv > 64) return fail(MODA_ERR_UNSUPPORTED, "query heads per KV head must be <= 64");
  // index arithmetic in the kernels uses 32-bit tile/row counts and 64-bit offsets
  const long long rows = 1LL * B * Hq * T;
  if (rows > (1LL << 31) || 1LL * B * Hkv > 65535 || T > (1 << 30) || L > 65535)
    return fail(MODA_ERR_UNSUPPORTED, "problem too large for the kernels' index ranges");
  return MODA_OK;
}

// Device check, cached per device: compute capability 10.x (B200 / sm_100a).
moda_status_t check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess)
    return fail(MODA_ERR_CUDA, "cudaGetDevice failed (no CUDA device?)");
  static std::mutex mu;
  static int known[64] = {0};  // 0 unknown, 1 ok, 2 unsupported
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return fail(MODA_ERR_UNSUPPORTED, "device index out of range");
  if (known[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return fail(MODA_ERR_CUDA, "cudaDeviceGetAttribute failed");
    known[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  if (known[dev] != 1)
    return fail(MODA_ERR_UNSUPPORTED, "the kernels are built for sm_100a (B200) only");
  return MODA_OK;
}

// Host-side fault injection, for testing how callers handle the library's errors; no
// kernel is launched in either mode.  The environment variable MODA_FAULT_INJECT is read
// on every call (so a test can set and clear it in-process):
//   validate  every compute entry point returns MODA_ERR_INVALID_ARGUMENT before its
//             argument checks;
//   launch    it returns MODA_ERR_CUDA once its argument checks have passed, in place of
//             the device query and the launch.
// Any other value, or none, injects nothing.
enum { kInjectNone = 0, kInjectValidate = 1, kInjectLaunch = 2 };

int fault_injection() {
  const char* e = getenv("MODA_FAULT_INJECT");
  if (e == nullptr) return kInjectNone;
  if (strcmp(e, "validate") == 0) return kInjectValidate;
  if (strcmp(e, "launch") == 0) return kInjectLaunch;
  return kInjectNone;
}

moda_status_t injected_at_validate() {
  if (fault_injection() == kInjectValidate)
    return fail(MODA_ERR_INVALID_ARGUMENT, "injected failure (MODA_FAULT_INJECT=validate)");
  return MODA_OK;
}

moda_status_t injected_at_launch() {
  if (fault_injection() == kInjectLaunch)
    return fail(MODA_ERR_CUDA, "injected failure (MODA_FAULT_INJECT=launch)");
  return MODA_OK;
}

moda::EncodeTiledFn get_encoder() {
  static std::once_flag once;
  static moda::EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<moda::EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

extern "C" {

const char* moda_status_string(moda_status_t status) {
  switch (status) {
    case MODA_OK: return "success";
    case MODA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case MODA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MODA_ERR_CUDA: return "CUDA error";
    case MODA_ERR_TIMEOUT: return "kernel wait timed out";
    case MODA_ERR_INTERNAL: return "kernel internal check failed";
  }
  return "unknown status";
}

const char* moda_last_error_message(void) { return g_msg; }

static moda_status_t forward_entry(const void* q, const void* k, const void* v,
                                   const void* kd, const void* vd, void* out, float* lse,
                                   int B, int Hq, int Hkv, int T, int L, int d, float scale,
                                   int causal, int depth_path, int depth_only,
                                   moda_stream_t stream) {
  g_msg[0] = 0;
  moda_status_t s = injected_at_validate();
  if (s != MODA_OK) return s;
  s = check_sizes(B, Hq, Hkv, T, L, d);
  if (s != MODA_OK) return s;
  if (depth_only) {
    if (L < 1) return fail(MODA_ERR_INVALID_ARGUMENT, "depth-only attention needs L >= 1");
    // no sequence keys; the kernel's K/V tensor maps are described over q and never read
    k = v = q;
  }
  if (depth_path < moda::kDepthPathAuto || depth_path > moda::kDepthPathDense)
    return fail(MODA_ERR_INVALID_ARGUMENT, "depth_path must be 0, 1 or 2");
  if (!q || !k || !v || !out || !lse)
    return fail(MODA_ERR_INVALID_ARGUMENT, "q, k, v, out and lse must be non-NULL");
  if (L > 0 && (!kd || !vd))
    return fail(MODA_ERR_INVALID_ARGUMENT, "kd and vd must be non-NULL when L > 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(lse) || (L > 0 && (!aligned16(kd) || !aligned16(vd))))
    return fail(MODA_ERR_INVALID_ARGUMENT, "every tensor pointer must be 16-byte aligned");
  if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
    return fail(MODA_ERR_INVALID_ARGUMENT, "scale must be finite");
  const size_t nq = size_t(B) * Hq * T * d * 2, nk = size_t(B) * Hkv * T * d * 2;
  const size_t nd = nk * size_t(L), nl = size_t(B) * Hq * T * 4;
  const void* ins[5] = {q, k, v, kd, vd};
  const size_t insz[5] = {nq, nk, nk, nd, nd};
  for (int i = 0; i < 5; ++i)
    if (overlaps(out, nq, ins[i], insz[i]) || overlaps(lse, nl, ins[i], insz[i]))
      return fail(MODA_ERR_INVALID_ARGUMENT, "out/lse must not overlap an input");
  if (overlaps(out, nq, lse, nl))
    return fail(MODA_ERR_INVALID_ARGUMENT, "out and lse must not overlap");
  moda::Problem p{B, Hq, Hkv, T, L, d, Hq / Hkv, causal ? 1 : 0, scale};
  p.depth_only = depth_only ? 1 : 0;
  if (depth_path == moda::kDepthPathDense && !moda::dense_depth_supported(p))
    return fail(MODA_ERR_UNSUPPORTED, "dense depth blocks need Hq/Hkv to divide 128");
  s = injected_at_launch();
  if (s != MODA_OK) return s;
  s = check_device();
  if (s != MODA_OK) return s;
  moda::EncodeTiledFn enc = get_encoder();
  if (!enc) return fail(MODA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  const char* why = "";
  cudaError_t e = moda::launch_forward(p, q, k, v, kd, vd, out, lse, depth_path, enc,
                                       static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) {
    snprintf(g_msg, sizeof(g_msg), "%s: %s", why, cudaGetErrorString(e));
    return MODA_ERR_CUDA;
  }
  return MODA_OK;
}

moda_status_t moda_forward(const void* q, const void* k, const void* v, const void* kd,
                           const void* vd, void* out, float* lse, int B, int Hq, int Hkv,
                           int T, int L, int d, float scale, int causal,
                           moda_stream_t stream) {
  return forward_entry(q, k, v, kd, vd, out, lse, B, Hq, Hkv, T, L, d, scale, causal,
                       moda::kDepthPathAuto, 0, stream);
}

moda_status_t moda_depth_attention_forward(const void* q, const void* kd, const void* vd,
                                           void* out, float* lse, int B, int Hq, int Hkv,
                                           int T, int L, int d, float scale,
                                           moda_stream_t stream) {
  return forward_entry(q, nullptr, nullptr, kd, vd, out, lse, B, Hq, Hkv, T, L, d, scale, 1,
                       moda::kDepthPathAuto, 1, stream);
}

moda_status_t moda_forward_depth_path(const void* q, const void* k, const void* v,
                                      const void* kd, const void* vd, void* out, float* lse,
                                      int B, int Hq, int Hkv, int T, int L, int d,
                                      float scale, int causal, int depth_path,
                                      moda_stream_t stream) {
  return forward_entry(q, k, v, kd, vd, out, lse, B, Hq, Hkv, T, L, d, scale, causal,
                       depth_path, 0, stream);
}

size_t moda_decode_workspace_size(int B, int Hq, int Hkv, int S, int L, int d) {
  if (check_sizes(B, Hq, Hkv, S, L, d) != MODA_OK) return 0;
  moda::Problem p{B, Hq, Hkv, S, L, d, Hq / Hkv, 1, 1.f};
  return moda::decode_workspace_bytes(p);
}

moda_status_t moda_decode(const void* q, const void* k, const void* v, const void* kd,
                          const void* vd, void* out, float* lse, void* workspace,
                          size_t workspace_bytes, int B, int Hq, int Hkv, int S, int L, int d,
                          float scale, moda_stream_t stream) {
  g_msg[0] = 0;
  moda_status_t s = injected_at_validate();
  if (s != MODA_OK) return s;
  s = check_sizes(B, Hq, Hkv, S, L, d);
  if (s != MODA_OK) return s;
  if (!q || !k || !v || !out || !lse || !workspace)
    return fail(MODA_ERR_INVALID_ARGUMENT, "q, k, v, out, lse and workspace must be non-NULL");
  if (L > 0 && (!kd || !vd))
    return fail(MODA_ERR_INVALID_ARGUMENT, "kd and vd must be non-NULL when L > 0");
  const void* all[8] = {q, k, v, kd, vd, out, lse, workspace};
  for (int i = 0; i < 8; ++i)
    if (all[i] && !aligned16(all[i]))
      return fail(MODA_ERR_INVALID_ARGUMENT, "every pointer must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(MODA_ERR_INVALID_ARGUMENT, "workspace must be 256-byte aligned");
  if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
    return fail(MODA_ERR_INVALID_ARGUMENT, "scale must be finite");
  moda::Problem p{B, Hq, Hkv, S, L, d, Hq / Hkv, 1, scale};
  const size_t need = moda::decode_workspace_bytes(p);
  if (workspace_bytes < need)
    return fail(MODA_ERR_INVALID_ARGUMENT, "workspace is smaller than moda_decode_workspace_size()");
  const size_t nq = size_t(B) * Hq * d * 2, nk = size_t(B) * Hkv * S * d * 2;
  const size_t nd = size_t(B) * Hkv * L * d * 2, nl = size_t(B) * Hq * 4;
  const void* ins[5] = {q, k, v, kd, vd};
  const size_t insz[5] = {nq, nk, nk, nd, nd};
  void* outs[3] = {out, lse, workspace};
  const size_t outsz[3] = {nq, nl, need};
  for (int o = 0; o < 3; ++o) {
    for (int i = 0; i < 5; ++i)
      if (overlaps(outs[o], outsz[o], ins[i], insz[i]))
        return fail(MODA_ERR_INVALID_ARGUMENT, "out/lse/workspace must not overlap an input");
    for (int o2 = o + 1; o2 < 3; ++o2)
      if (overlaps(outs[o], outsz[o], outs[o2], outsz[o2]))
        return fail(MODA_ERR_INVALID_ARGUMENT, "out, lse and workspace must not overlap");
  }
  s = injected_at_launch();
  if (s != MODA_OK) return s;
  s = check_device();
  if (s != MODA_OK) return s;
  moda::EncodeTiledFn enc = get_encoder();
  if (!enc) return fail(MODA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  const char* why = "";
  cudaError_t e = moda::launch_decode(p, q, k, v, kd, vd, out, lse, workspace, enc,
                                      static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) {
    snprintf(g_msg, sizeof(g_msg), "%s: %s", why, cudaGetErrorString(e));
    return MODA_ERR_CUDA;
  }
  return MODA_OK;
}

moda_status_t moda_depth_kv_write(const void* x, const void* w, void* kd, void* vd, int B,
                                  int T, int hidden, int Hkv, int d, int L, int slot,
                                  moda_stream_t stream) {
  g_msg[0] = 0;
  if (injected_at_validate() != MODA_OK) return MODA_ERR_INVALID_ARGUMENT;
  if (B < 1 || T < 1 || hidden < 1 || Hkv < 1 || L < 1)
    return fail(MODA_ERR_INVALID_ARGUMENT, "B, T, hidden, Hkv and L must be positive");
  if (slot < 0 || slot >= L) return fail(MODA_ERR_INVALID_ARGUMENT, "slot must lie in [0, L)");
  if (d != 64 && d != 128) return fail(MODA_ERR_UNSUPPORTED, "d must be 64 or 128");
  if ((Hkv * d) % 128 != 0)
    return fail(MODA_ERR_UNSUPPORTED, "Hkv * d must be a multiple of 128");
  if (hidden % 8 != 0)
    return fail(MODA_ERR_UNSUPPORTED, "hidden must be a multiple of 8 (16-byte rows)");
  // the kernel indexes the B*T tokens with 32-bit integers
  if (1LL * B * T > (1LL << 31) - 256)
    return fail(MODA_ERR_UNSUPPORTED, "B*T is too large for the kernel's token index");
  if (!x || !w || !kd || !vd)
    return fail(MODA_ERR_INVALID_ARGUMENT, "x, w, kd and vd must be non-NULL");
  if (!aligned16(x) || !aligned16(w) || !aligned16(kd) || !aligned16(vd))
    return fail(MODA_ERR_INVALID_ARGUMENT, "every pointer must be 16-byte aligned");
  const size_t nx = size_t(B) * T * hidden * 2, nw = size_t(2) * Hkv * d * hidden * 2;
  const size_t nd = size_t(B) * Hkv * T * L * d * 2;
  if (overlaps(kd, nd, x, nx) || overlaps(kd, nd, w, nw) || overlaps(vd, nd, x, nx) ||
      overlaps(vd, nd, w, nw) || overlaps(kd, nd, vd, nd))
    return fail(MODA_ERR_INVALID_ARGUMENT, "kd/vd must not overlap x, w or each other");
  moda_status_t s = injected_at_launch();
  if (s != MODA_OK) return s;
  s = check_device();
  if (s != MODA_OK) return s;
  moda::EncodeTiledFn enc = get_encoder();
  if (!enc) return fail(MODA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  moda::KvWriteProblem p{B, T, hidden, Hkv, d, L, slot};
  const char* why = "";
  cudaError_t e = moda::launch_kvwrite(p, x, w, kd, vd, enc, static_cast<cudaStream_t>(stream),
                                       &why);
  if (e != cudaSuccess) {
    snprintf(g_msg, sizeof(g_msg), "%s: %s", why, cudaGetErrorString(e));
    return MODA_ERR_CUDA;
  }
  return MODA_OK;
}

size_t moda_backward_workspace_size(int B, int Hq, int Hkv, int T, int L, int d) {
  if (check_sizes(B, Hq, Hkv, T, L, d) != MODA_OK) return 0;
  moda::Problem p{B, Hq, Hkv, T, L, d, Hq / Hkv, 1, 1.f};
  return moda::backward_workspace_bytes(p);
}

}  // extern "C"

namespace {

// validate_only: run the argument checks that need neither the workspace nor the device
// and return (no device query, no launch); the workspace may then be NULL.
moda_status_t backward_entry(const void* q, const void* k, const void* v, const void* kd,
                             const void* vd, const void* out, const float* lse,
                             const void* dout, void* dq, void* dk, void* dv, void* dkd,
                             void* dvd, void* workspace, size_t workspace_bytes, int B,
                             int Hq, int Hkv, int T, int L, int d, float scale, int causal,
                             unsigned stages, int depth_only, moda_stream_t stream,
                             bool validate_only = false) {
  g_msg[0] = 0;
  moda_status_t s = injected_at_validate();
  if (s != MODA_OK) return s;
  s = check_sizes(B, Hq, Hkv, T, L, d);
  if (s != MODA_OK) return s;
  if (depth_only) {
    if (L < 1) return fail(MODA_ERR_INVALID_ARGUMENT, "depth-only attention needs L >= 1");
    k = v = nullptr;  // no sequence keys: k, v, dk, dv are not used
    dk = dv = nullptr;
    stages = moda::kStageDepth | moda::kStageConvert;
  }
  if (!q || !out || !lse || !dout || !dq || (!workspace && !validate_only) ||
      (!depth_only && (!k || !v || !dk || !dv)))
    return fail(MODA_ERR_INVALID_ARGUMENT,
                "q, k, v, out, lse, dout, dq, dk, dv and workspace must be non-NULL");
  if (L > 0 && (!kd || !vd || !dkd || !dvd))
    return fail(MODA_ERR_INVALID_ARGUMENT, "kd, vd, dkd and dvd must be non-NULL when L > 0");
  const void* all[14] = {q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd, workspace};
  for (int i = 0; i < 14; ++i)
    if (all[i] && !aligned16(all[i]))
      return fail(MODA_ERR_INVALID_ARGUMENT, "every pointer must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(MODA_ERR_INVALID_ARGUMENT, "workspace must be 256-byte aligned");
  if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
    return fail(MODA_ERR_INVALID_ARGUMENT, "scale must be finite");
  moda::Problem p{B, Hq, Hkv, T, L, d, Hq / Hkv, causal ? 1 : 0, scale};
  p.depth_only = depth_only ? 1 : 0;
  if (validate_only) {
    // the checks of the gradient buffers against the inputs and each other
    const size_t nq = size_t(B) * Hq * T * d * 2, nk = size_t(B) * Hkv * T * d * 2;
    const size_t nd = nk * size_t(L), nl = size_t(B) * Hq * T * 4;
    const void* ins[8] = {q, k, v, kd, vd, out, lse, dout};
    const size_t insz[8] = {nq, nk, nk, nd, nd, nq, nl, nq};
    void* outs[5] = {dq, dk, dv, dkd, dvd};
    const size_t outsz[5] = {nq, nk, nk, nd, nd};
    for (int o = 0; o < 5; ++o) {
      for (int i = 0; i < 8; ++i)
        if (overlaps(outs[o], outsz[o], ins[i], insz[i]))
          return fail(MODA_ERR_INVALID_ARGUMENT, "gradient buffers must not overlap an input");
      for (int o2 = o + 1; o2 < 5; ++o2)
        if (overlaps(outs[o], outsz[o], outs[o2], outsz[o2]))
          return fail(MODA_ERR_INVALID_ARGUMENT, "gradient buffers must not overlap each other");
    }
    return MODA_OK;
  }
  const size_t need = moda::backward_workspace_bytes(p);
  if (workspace_bytes < need)
    return fail(MODA_ERR_INVALID_ARGUMENT, "workspace is smaller than moda_backward_workspace_size()");
  const size_t nq = size_t(B) * Hq * T * d * 2, nk = size_t(B) * Hkv * T * d * 2;
  const size_t nd = nk * size_t(L), nl = size_t(B) * Hq * T * 4;  // (k, v unused: NULL)
  const void* ins[8] = {q, k, v, kd, vd, out, lse, dout};
  const size_t insz[8] = {nq, nk, nk, nd, nd, nq, nl, nq};
  void* outs[6] = {dq, dk, dv, dkd, dvd, workspace};
  const size_t outsz[6] = {nq, nk, nk, nd, nd, need};
  for (int o = 0; o < 6; ++o) {
    for (int i = 0; i < 8; ++i)
      if (overlaps(outs[o], outsz[o], ins[i], insz[i]))
        return fail(MODA_ERR_INVALID_ARGUMENT, "gradient/workspace buffers must not overlap an input");
    for (int o2 = o + 1; o2 < 6; ++o2)
      if (overlaps(outs[o], outsz[o], outs[o2], outsz[o2]))
        return fail(MODA_ERR_INVALID_ARGUMENT, "gradient/workspace buffers must not overlap each other");
  }
  s = injected_at_launch();
  if (s != MODA_OK) return s;
  s = check_device();
  if (s != MODA_OK) return s;
  moda::EncodeTiledFn enc = get_encoder();
  if (!enc) return fail(MODA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  const char* why = "";
  cudaError_t e = moda::launch_backward(p, q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd,
                                        dvd, workspace, stages, enc,
                                        static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) {
    snprintf(g_msg, sizeof(g_msg), "%s: %s", why, cudaGetErrorString(e));
    return MODA_ERR_CUDA;
  }
  return MODA_OK;
}

}  // namespace

extern "C" {

moda_status_t moda_backward(const void* q, const void* k, const void* v, const void* kd,
                            const void* vd, const void* out, const float* lse,
                            const void* dout, void* dq, void* dk, void* dv, void* dkd,
                            void* dvd, void* workspace, size_t workspace_bytes, int B,
                            int Hq, int Hkv, int T, int L, int d, float scale, int causal,
                            moda_stream_t stream) {
  return backward_entry(q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd, workspace,
                        workspace_bytes, B, Hq, Hkv, T, L, d, scale, causal, moda::kStagesAll,
                        0, stream);
}

moda_status_t moda_backward_stages(const void* q, const void* k, const void* v,
                                   const void* kd, const void* vd, const void* out,
                                   const float* lse, const void* dout, void* dq, void* dk,
                                   void* dv, void* dkd, void* dvd, void* workspace,
                                   size_t workspace_bytes, int B, int Hq, int Hkv, int T,
                                   int L, int d, float scale, int causal, unsigned stages,
                                   moda_stream_t stream) {
  if (stages == 0 || (stages & ~moda::kStagesAll)) {
    g_msg[0] = 0;
    return fail(MODA_ERR_INVALID_ARGUMENT, "stages must be a non-empty subset of {1, 2, 4}");
  }
  return backward_entry(q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd, workspace,
                        workspace_bytes, B, Hq, Hkv, T, L, d, scale, causal, stages, 0,
                        stream);
}

moda_status_t moda_depth_attention_backward(const void* q, const void* kd, const void* vd,
                                            const void* out, const float* lse,
                                            const void* dout, void* dq, void* dkd, void* dvd,
                                            void* workspace, size_t workspace_bytes, int B,
                                            int Hq, int Hkv, int T, int L, int d, float scale,
                                            moda_stream_t stream) {
  return backward_entry(q, nullptr, nullptr, kd, vd, out, lse, dout, dq, nullptr, nullptr,
                        dkd, dvd, workspace, workspace_bytes, B, Hq, Hkv, T, L, d, scale, 1,
                        moda::kStagesAll, 1, stream);
}

moda_status_t moda_test_set_device_fault(int fault, uint64_t wait_limit_ns) {
  g_msg[0] = 0;
  if (fault < 0 || fault > moda::kFaultForwardNoLoads)
    return fail(MODA_ERR_INVALID_ARGUMENT, "fault must be 0 (none) or 1 (forward issues no loads)");
  if (wait_limit_ns != 0 && (wait_limit_ns < 100000ull || wait_limit_ns > 10000000000ull))
    return fail(MODA_ERR_INVALID_ARGUMENT, "wait_limit_ns must be 0 or lie in [1e5, 1e10]");
  moda_status_t s = check_device();
  if (s != MODA_OK) return s;
  const uint64_t limit = wait_limit_ns ? wait_limit_ns : moda::kWaitLimitNs;
  cudaError_t e = cudaMemcpyToSymbol(moda::g_wait_limit_ns, &limit, sizeof(limit));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(moda::g_device_fault, &fault, sizeof(fault));
  if (e != cudaSuccess)
    return fail(MODA_ERR_CUDA, "setting the test knobs failed: %s", cudaGetErrorString(e));
  return MODA_OK;
}

moda_status_t moda_test_exp2_fma(const float* x, float* y, int n, moda_stream_t stream) {
  g_msg[0] = 0;
  if (n < 0 || n > (1 << 30))
    return fail(MODA_ERR_INVALID_ARGUMENT, "n must lie in [0, 2^30]");
  if (n > 0 && (x == nullptr || y == nullptr))
    return fail(MODA_ERR_INVALID_ARGUMENT, "x and y must be non-NULL when n > 0");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 3u)
    return fail(MODA_ERR_INVALID_ARGUMENT, "x and y must be 4-byte aligned");
  moda_status_t s = check_device();
  if (s != MODA_OK) return s;
  const cudaError_t e =
      moda::launch_test_exp2_fma(x, y, n, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return fail(MODA_ERR_CUDA, "exp2 test kernel launch failed: %s", cudaGetErrorString(e));
  return MODA_OK;
}

moda_status_t moda_check_device_errors(moda_stream_t stream, uint32_t* flags) {
  g_msg[0] = 0;
  if (flags) *flags = 0;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return fail(MODA_ERR_CUDA, "stream synchronisation failed: %s", cudaGetErrorString(e));
  uint32_t word = 0;
  const uint32_t zero = 0;
  e = cudaMemcpyFromSymbol(&word, moda::g_error_word, sizeof(word));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(moda::g_error_word, &zero, sizeof(zero));
  if (e != cudaSuccess)
    return fail(MODA_ERR_CUDA, "reading the kernel error word failed: %s", cudaGetErrorString(e));
  if (flags) *flags = word;
  if (word & 1u) return fail(MODA_ERR_TIMEOUT, "a kernel's bounded wait ran out");
  if (word & 2u) return fail(MODA_ERR_INTERNAL, "a kernel's internal check failed");
  return MODA_OK;
}

}  // extern "C"
