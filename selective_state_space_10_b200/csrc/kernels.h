// kernels.h -- host-side launchers of the libssd kernels (internal to the library).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace ssd {

// prefill_simt.cu
cudaError_t launch_dA_cumsum(const float *dt, const float *A, float *cum, const Dims &d, int Q, int nc,
                             cudaStream_t st);
template <typename T>
cudaError_t launch_chunk_state_simt(const T *x, const float *dt, const T *B, const float *cum, float *states,
                                    const Dims &d, int Q, int nc, cudaStream_t st);
// init: state before the first token (NULL: zero); cstates: state after each chunk (NULL: not written)
cudaError_t launch_state_passing(float *states, const float *cum, const float *init, float *final_state,
                                 float *cstates, const Dims &d, int Q, int nc, cudaStream_t st);
template <typename T>
cudaError_t launch_chunk_scan_simt(const T *x, const float *dt, const T *B, const T *C, const float *D,
                                   const float *cum, const float *hprev, float *y, const Dims &d, int Q, int nc,
                                   cudaStream_t st);
size_t chunk_scan_simt_smem_bytes(int N);

// prefill_tc.cu (bf16 x/B/C, P = 64, N = 128, Q in {128, 256})
bool tc_prefill_supported(const Dims &d, int Q);
// floats of the per-(batch, head, chunk) decay table the tensor-core kernels share
size_t tc_prefill_table_floats(const Dims &d, int Q, int nc);
cudaError_t launch_tc_prefill(const __nv_bfloat16 *x, const float *dt, const float *A, const __nv_bfloat16 *B,
                              const __nv_bfloat16 *C, const float *D, const float *init, float *y, float *final_state,
                              float *cstates, float *tab, float *states, float *cdecay, __nv_bfloat16 *hprev, int *err,
                              const Dims &d, int Q, int nc, cudaStream_t st, const cudaEvent_t *ev);

// decode.cu
template <typename T>
cudaError_t launch_decode_step(float *state, const T *x, const float *dt, const float *A, const T *B,
                               const T *C, const float *D, float *y, const Dims &d, cudaStream_t st);

// frontend.cu: conv + SiLU + split, softplus dt; the new conv state when state_out != NULL
template <typename T>
cudaError_t launch_frontend(const T *xbc, const float *w, const float *bias, const float *state_in,
                            float *state_out, const float *dt_raw, const float *dt_bias, T *x, T *B, T *C, float *dt,
                            const Dims &d, cudaStream_t st);

// decode_window.cu (window length 1 .. 16)
template <typename T>
cudaError_t launch_decode_window_step(const float *state, T *win_x, float *win_dt, T *win_B, int W, int pos,
                                      const T *x, const float *dt, const float *A, const T *B, const T *C,
                                      const float *D, float *y, const Dims &d, cudaStream_t st);
template <typename T>
cudaError_t launch_decode_window_flush(float *state, const T *win_x, const float *win_dt, const T *win_B, int W,
                                       int count, const float *A, const Dims &d, cudaStream_t st);

}  // namespace ssd
