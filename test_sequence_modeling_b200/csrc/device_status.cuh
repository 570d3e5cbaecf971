// device_status.cuh - the library's device status word.
//
// A kernel whose bounded wait expires records its error code here (first
// writer wins) instead of trapping, so that the context stays usable and the
// host can read the code back with ttt_last_device_status().
#pragma once

namespace ttt {

__device__ int g_device_status = 0;

__device__ __forceinline__ void record_device_error(int code) {
  atomicCAS(&g_device_status, 0, code);
}

}  // namespace ttt
