// prefill_tc.cuh -- tensor-core (tcgen05) chunked prefill for bf16, dk = dv = 128.
#pragma once

#include "common.cuh"

namespace kda {

constexpr bool kTcPathReady = false;

inline size_t tc_slot_bytes() { return 0; }

inline cudaError_t launch_tc_prefill(const void*, const void*, const void*, const float*, const float*, const float*,
                                     float*, void*, const WsHeader*, const int*, const int32_t*, int, int, int, int,
                                     char*, cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace kda
