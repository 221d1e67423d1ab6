// internal.h -- what flce_api.cu shares with the library's other translation
// units: launch accounting and profiling hooks, kernel kinds, and launchers
// for the small integer / reduction kernels every entry point uses.  Not part
// of the C ABI.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace flce_internal {

// Kernel kinds reported by flce_profile_stop / flce_kernel_name, beyond the
// ones flce_api.cu launches itself.
enum : int32_t { kKindCeForward = 19, kKindCeBackward = 20, kKindCeFused = 21 };

// Profiling events around one launch (no-ops unless flce_profile_start ran);
// prof_after also counts the launch for flce_last_launch_count.
void prof_before(cudaStream_t st);
void prof_after(cudaStream_t st, int32_t kind);
// Start counting the launches of a new entry-point call on this host thread.
void reset_launch_count();
// The process-wide bound on every wait inside the kernels (flce_set_wait_limit_ns).
unsigned long long wait_limit_ns();
// Streaming multiprocessors of the current device (0 if it cannot be read).
int device_sm_count();

// labels check + N_valid into the workspace header (status word reset).
cudaError_t launch_labels(const int64_t* labels, int64_t BT, int64_t V, int64_t ignore_index,
                          void* ws, cudaStream_t st);
// The op's own shifted copy of token ids (shift_seq_len = T > 0).
cudaError_t launch_shift(const int64_t* ids, int64_t BT, int64_t T, int64_t ignore_index,
                         int64_t* out, cudaStream_t st);
// loss = fp64 fixed-order sum of row_loss / N_valid (0 when N_valid = 0).
cudaError_t launch_finalize(const float* row_loss, int64_t BT, const void* ws, float* loss,
                            cudaStream_t st);

}  // namespace flce_internal
