// flce_ce.cu -- C ABI of the cross-entropy path for callers that already
// hold the logits (flce_ce_forward / flce_ce_backward, declared and
// documented in include/flce.h).
//
// Launch sequence:
//   forward   [shift_labels] -> labels_kernel (status, N_valid) ->
//             ce_forward_kernel (lse, per-row NLL) -> finalize_kernel (loss)
//   backward  [shift_labels] -> labels_kernel -> ce_backward_kernel (dlogits)
// The backward reads the logits again and rebuilds the softmax from them and
// the forward's lse (PyTorch PR #126348, point b.); nothing of size BT x V is
// written except the gradient the caller asked for.
#include <cmath>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "flce.h"
#include "internal.h"
#include "ce_kernels.cuh"

using namespace flce;
using namespace flce_internal;

namespace {

constexpr size_t kHeaderBytes = 256;
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool softcap_on(float c) { return c > 0.f && std::isfinite(c); }
bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }
size_t elem_size(int32_t dtype) { return dtype == FLCE_BF16 ? 2 : 4; }
int64_t ld_of(int64_t ld, int64_t V) { return ld == 0 ? V : ld; }

flce_status_t check_ce(const flce_ce_problem_t* p) {
  if (!p) return FLCE_ERR_INVALID_ARG;
  if (p->reserved1 != 0 || p->shift_seq_len < 0) return FLCE_ERR_INVALID_ARG;
  if (p->BT < 0 || p->V <= 0 || p->ld < 0 || p->ld_grad < 0) return FLCE_ERR_INVALID_ARG;
  if (p->shift_seq_len > 0 && p->BT % p->shift_seq_len != 0) return FLCE_ERR_INVALID_ARG;
  if (p->dtype != FLCE_BF16 && p->dtype != FLCE_FP32) return FLCE_ERR_UNSUPPORTED;
  if (p->BT >= (int64_t(1) << 31) || p->V >= (int64_t(1) << 31)) return FLCE_ERR_UNSUPPORTED;
  if (ld_of(p->ld, p->V) < p->V || ld_of(p->ld_grad, p->V) < p->V) return FLCE_ERR_INVALID_ARG;
  if (ld_of(p->ld, p->V) >= (int64_t(1) << 40) || ld_of(p->ld_grad, p->V) >= (int64_t(1) << 40))
    return FLCE_ERR_UNSUPPORTED;
  return FLCE_OK;
}

struct CePlan {
  size_t off_rowloss = 0, off_shift = 0, total = 0;
};

void make_ce_plan(const flce_ce_problem_t* p, int op, CePlan* pl) {
  size_t off = kHeaderBytes;
  const size_t rows = size_t(p->BT);
  if (op == FLCE_OP_FORWARD || op == FLCE_OP_FUSED) {
    pl->off_rowloss = off;
    off = align256(off + rows * 4);
  }
  if (p->shift_seq_len > 0) {
    pl->off_shift = off;
    off = align256(off + rows * 8);
  }
  pl->total = off;
}

// Common checks and the labels prologue; on success *labels_out is the
// labels array the kernels read (the op's shifted copy when shifting).
flce_status_t prologue(const flce_ce_problem_t* p, int op, const void* logits,
                       const int64_t* labels, void* ws, size_t ws_bytes, cudaStream_t st,
                       CePlan* pl, const int64_t** labels_out) {
  flce_status_t s = check_ce(p);
  if (s != FLCE_OK) return s;
  if (!ws || (p->BT > 0 && (!logits || !labels))) return FLCE_ERR_INVALID_ARG;
  if (!aligned(ws, 256) || !aligned(labels, 8) || !aligned(logits, elem_size(p->dtype)))
    return FLCE_ERR_MISALIGNED;
  make_ce_plan(p, op, pl);
  if (ws_bytes < pl->total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* w = static_cast<uint8_t*>(ws);
  *labels_out = labels;
  if (p->shift_seq_len > 0) {
    int64_t* sh = reinterpret_cast<int64_t*>(w + pl->off_shift);
    if (launch_shift(labels, p->BT, p->shift_seq_len, p->ignore_index, sh, st) != cudaSuccess)
      return FLCE_ERR_CUDA;
    *labels_out = sh;
  }
  if (launch_labels(*labels_out, p->BT, p->V, p->ignore_index, ws, st) != cudaSuccess)
    return FLCE_ERR_CUDA;
  return FLCE_OK;
}

template <typename T>
cudaError_t launch_ce_forward(const flce_ce_problem_t* p, const void* logits,
                              const int64_t* labels, float* lse, float* rowloss, const void* ws,
                              cudaStream_t st) {
  const T* Z = static_cast<const T*>(logits);
  const WsHeader* hdr = static_cast<const WsHeader*>(ws);
  const int64_t ld = ld_of(p->ld, p->V);
  prof_before(st);
  if (softcap_on(p->softcap))
    ce_forward_kernel<T, true><<<unsigned(p->BT), kCeThreads, 0, st>>>(
        Z, ld, p->V, labels, p->ignore_index, p->softcap, lse, rowloss, hdr);
  else
    ce_forward_kernel<T, false><<<unsigned(p->BT), kCeThreads, 0, st>>>(
        Z, ld, p->V, labels, p->ignore_index, 0.f, lse, rowloss, hdr);
  prof_after(st, kKindCeForward);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ce_backward(const flce_ce_problem_t* p, const void* logits,
                               const int64_t* labels, const float* lse, const float* dloss,
                               void* dlogits, const void* ws, cudaStream_t st) {
  const T* Z = static_cast<const T*>(logits);
  T* dZ = static_cast<T*>(dlogits);
  const WsHeader* hdr = static_cast<const WsHeader*>(ws);
  const int64_t ld = ld_of(p->ld, p->V), ldg = ld_of(p->ld_grad, p->V);
  prof_before(st);
  if (softcap_on(p->softcap))
    ce_backward_kernel<T, true><<<unsigned(p->BT), kCeThreads, 0, st>>>(
        Z, ld, dZ, ldg, p->V, labels, p->ignore_index, p->softcap, lse, dloss, hdr);
  else
    ce_backward_kernel<T, false><<<unsigned(p->BT), kCeThreads, 0, st>>>(
        Z, ld, dZ, ldg, p->V, labels, p->ignore_index, 0.f, lse, dloss, hdr);
  prof_after(st, kKindCeBackward);
  return cudaGetLastError();
}

template <typename T, bool CAP>
cudaError_t launch_ce_fused_t(const flce_ce_problem_t* p, const void* logits,
                              const int64_t* labels, float dloss, float* lse, float* rowloss,
                              void* dlogits, void* ws, cudaStream_t st) {
  const T* Z = static_cast<const T*>(logits);
  T* dZ = static_cast<T*>(dlogits);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  const int64_t ld = ld_of(p->ld, p->V), ldg = ld_of(p->ld_grad, p->V);
  const float cap = CAP ? p->softcap : 0.f;
  const size_t row_bytes = size_t(p->V) * sizeof(T);
  cudaError_t e;
  if (row_bytes <= size_t(kCeFusedRowMax)) {
    // Two row buffers per persistent block, one block per SM: a producer
    // warp and kCePipeWarps compute warps.
    const uint32_t buf = uint32_t((row_bytes + 15) / 16 * 16);
    auto kern = ce_fused_pipe_kernel<T, CAP>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(2 * buf))) != cudaSuccess)
      return e;
    int grid = device_sm_count();
    if (grid <= 0) return cudaErrorInvalidDevice;
    if (int64_t(grid) > p->BT) grid = int(p->BT);
    prof_before(st);
    kern<<<unsigned(grid), kCePipeThreads, 2 * buf, st>>>(
        Z, ld, dZ, ldg, p->BT, p->V, labels, p->ignore_index, cap, dloss, lse, rowloss, hdr,
        buf, wait_limit_ns());
  } else {
    prof_before(st);
    ce_fused_rows_kernel<T, CAP><<<unsigned(p->BT), kCeFusedThreads, 0, st>>>(
        Z, ld, dZ, ldg, p->V, labels, p->ignore_index, cap, dloss, lse, rowloss, hdr);
  }
  prof_after(st, kKindCeFused);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ce_fused(const flce_ce_problem_t* p, const void* logits, const int64_t* labels,
                            float dloss, float* lse, float* rowloss, void* dlogits, void* ws,
                            cudaStream_t st) {
  return softcap_on(p->softcap)
             ? launch_ce_fused_t<T, true>(p, logits, labels, dloss, lse, rowloss, dlogits, ws, st)
             : launch_ce_fused_t<T, false>(p, logits, labels, dloss, lse, rowloss, dlogits, ws,
                                           st);
}

}  // namespace

extern "C" {

size_t flce_ce_workspace_size(const flce_ce_problem_t* p, int op) {
  if (check_ce(p) != FLCE_OK) return 0;
  if (op != FLCE_OP_FORWARD && op != FLCE_OP_BACKWARD && op != FLCE_OP_FUSED) return 0;
  CePlan pl;
  make_ce_plan(p, op, &pl);
  return pl.total;
}

flce_status_t flce_ce_forward(const flce_ce_problem_t* p, const void* logits,
                              const int64_t* labels, float* loss, float* lse, void* ws,
                              size_t ws_bytes, struct CUstream_st* stream) {
  reset_launch_count();
  flce_status_t s = check_ce(p);
  if (s != FLCE_OK) return s;
  if (!loss || (p->BT > 0 && !lse)) return FLCE_ERR_INVALID_ARG;
  if (!aligned(loss, 4) || !aligned(lse, 4)) return FLCE_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CePlan pl;
  const int64_t* lab = nullptr;
  if ((s = prologue(p, FLCE_OP_FORWARD, logits, labels, ws, ws_bytes, st, &pl, &lab)) != FLCE_OK)
    return s;
  float* rowloss = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.off_rowloss);
  if (p->BT > 0) {
    const cudaError_t e =
        p->dtype == FLCE_BF16
            ? launch_ce_forward<__nv_bfloat16>(p, logits, lab, lse, rowloss, ws, st)
            : launch_ce_forward<float>(p, logits, lab, lse, rowloss, ws, st);
    if (e != cudaSuccess) return FLCE_ERR_CUDA;
  }
  return launch_finalize(rowloss, p->BT, ws, loss, st) == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

flce_status_t flce_ce_backward(const flce_ce_problem_t* p, const void* logits,
                               const int64_t* labels, const float* lse, const float* dloss,
                               void* dlogits, void* ws, size_t ws_bytes,
                               struct CUstream_st* stream) {
  reset_launch_count();
  flce_status_t s = check_ce(p);
  if (s != FLCE_OK) return s;
  if (!dloss || (p->BT > 0 && (!lse || !dlogits))) return FLCE_ERR_INVALID_ARG;
  if (!aligned(dloss, 4) || !aligned(lse, 4) || !aligned(dlogits, elem_size(p->dtype)))
    return FLCE_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CePlan pl;
  const int64_t* lab = nullptr;
  if ((s = prologue(p, FLCE_OP_BACKWARD, logits, labels, ws, ws_bytes, st, &pl, &lab)) !=
      FLCE_OK)
    return s;
  if (p->BT == 0) return FLCE_OK;
  const cudaError_t e =
      p->dtype == FLCE_BF16
          ? launch_ce_backward<__nv_bfloat16>(p, logits, lab, lse, dloss, dlogits, ws, st)
          : launch_ce_backward<float>(p, logits, lab, lse, dloss, dlogits, ws, st);
  return e == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

}  // extern "C"

extern "C" flce_status_t flce_ce_fused(const flce_ce_problem_t* p, const void* logits,
                                       const int64_t* labels, float dloss, float* loss,
                                       float* lse, void* dlogits, void* ws, size_t ws_bytes,
                                       struct CUstream_st* stream) {
  reset_launch_count();
  flce_status_t s = check_ce(p);
  if (s != FLCE_OK) return s;
  if (!loss || (p->BT > 0 && !dlogits)) return FLCE_ERR_INVALID_ARG;
  if (!aligned(loss, 4) || !aligned(lse, 4) || !aligned(dlogits, elem_size(p->dtype)))
    return FLCE_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CePlan pl;
  const int64_t* lab = nullptr;
  if ((s = prologue(p, FLCE_OP_FUSED, logits, labels, ws, ws_bytes, st, &pl, &lab)) != FLCE_OK)
    return s;
  float* rowloss = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.off_rowloss);
  if (p->BT > 0) {
    const cudaError_t e =
        p->dtype == FLCE_BF16
            ? launch_ce_fused<__nv_bfloat16>(p, logits, lab, dloss, lse, rowloss, dlogits, ws, st)
            : launch_ce_fused<float>(p, logits, lab, dloss, lse, rowloss, dlogits, ws, st);
    if (e != cudaSuccess) return FLCE_ERR_CUDA;
  }
  return launch_finalize(rowloss, p->BT, ws, loss, st) == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}
