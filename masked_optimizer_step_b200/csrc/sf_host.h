// sf_host.h -- host-side helpers shared by the C-ABI entry points.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sf.h"

namespace sf {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(sf_stream s) { return reinterpret_cast<cudaStream_t>(s); }

// Returns SF_OK when the last launch succeeded, SF_ERR_CUDA otherwise (the sticky error state
// of the runtime is left for the caller to inspect).
inline int launch_status()
{
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SF_OK : SF_ERR_CUDA;
}

// A mask whose arrays are all present and whose sizes make sense.
inline int check_mask(const sf_mask &m)
{
    if (m.R <= 0 || (m.R & 31) || m.slot_cap < 0 || m.slot_cap > m.R) return SF_ERR_ARG;
    if (!m.charge || !m.accum || !m.words || !m.active_rows || !m.active_tiles || !m.tile_rows || !m.row_slot ||
        !m.counts || !m.slot_step || (!m.free_slots && m.slot_cap > 0))
        return SF_ERR_ARG;
    return SF_OK;
}

// Number of SMs of the current device (queried per call; cheap).
inline int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

}  // namespace sf
