// fa_host.h -- host-side pieces shared by the forward and backward launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_b200.h"  // include/ is on the include path

namespace fa {

// Properties of the current device that the launchers need.
struct DeviceInfo {
  int device;
  int sm_count;
  int max_smem_optin;
};

// FA_OK, or FA_ERR_DEVICE when the current device is not compute capability
// 10.0, or FA_ERR_LAUNCH when the runtime cannot be queried.
int current_device(DeviceInfo* info);

// FA_OK when e is cudaSuccess; otherwise records e (fa_last_cuda_error) and
// returns FA_ERR_LAUNCH.
int launch_status(cudaError_t e);

// FA_OK when the kernel was compiled with the register count its warpgroup
// register split assumes (kLaunchRegs a thread at 384 threads).
int check_launch_regs(const void* kernel);

// Counts kernel launches (fa_kernel_launches).
void note_launches(unsigned n);

// Takes (and disarms) the event pair armed for the next forward (bwd=false)
// or backward (bwd=true) main kernel; both are null when none is armed.
void take_kernel_events(bool bwd, cudaEvent_t* start, cudaEvent_t* stop);

// Device address of this library's status word on the current device.
unsigned long long* device_status_ptr();

// Tensor map over a contiguous [B, N, H, d] 16-bit tensor for TMA tile loads
// of `box_rows` tokens x 64 elements of one head (128 bytes, 128-byte swizzle).
// Rows past N are filled with zeros by the hardware.
int make_tmap_bnhd(CUtensorMap* map, const void* base, bool bf16, int B, int N, int H, int d,
                   int box_rows);

// Tensor map over a contiguous [rows, cols] fp32 matrix for TMA tiles of
// box_rows x box_cols (box_cols * 4 = 128 bytes, 128-byte swizzle).
int make_tmap_f32_rows(CUtensorMap* map, const void* base, size_t rows, int cols, int box_cols,
                       int box_rows);

// The backward entry points' argument checks (FA_OK or an FA_ERR_* code).
int check_bwd_args(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   float scale);

// Launchers (argument validation is done by the callers in fa_api.cu).
template <class T>
int fwd_launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int N, int d, float scale, cudaStream_t stream);
template <class T>
int bwd_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
               float scale, cudaStream_t stream);

}  // namespace fa
