// Per-device status word: OR of ENGRAM_STATUS_* bits raised by kernels that met bad data or
// gave up a bounded wait.  Read and cleared by engram_device_status().
#pragma once
#include <cstdint>

__device__ uint32_t g_engram_status = 0;
