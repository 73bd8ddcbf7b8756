// status.cuh -- the per-device status word kernels use to report errors.
//
// One int per device (a static __device__ variable of this shared library,
// which is built as a single translation unit). A kernel records the FIRST
// error only (atomicCAS from 0); attn_check() reads and clears it after
// synchronising the caller's stream.
#pragma once

namespace attn {

static __device__ int g_attn_device_status = 0;

__device__ __forceinline__ void record_status(int code) {
    atomicCAS(&g_attn_device_status, 0, code);
}

}  // namespace attn
