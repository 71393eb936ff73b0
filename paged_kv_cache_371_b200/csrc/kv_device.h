// Shared host-side helpers of the CUDA translation units.
#pragma once

#include <cuda_runtime.h>

// Device address of the current device's error word (bits KV_DEV_*), or
// nullptr if it cannot be resolved.
int* kv_error_word_ptr();

// KV_OK, or KV_ERR_CUDA with the error text recorded.
int kv_cuda_check(cudaError_t e, const char* where);
