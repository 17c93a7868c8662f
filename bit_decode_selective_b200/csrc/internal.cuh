// internal.cuh -- entry points shared between translation units of the library.
#pragma once

#include "common.cuh"

namespace sf {

sf_status check_select_args(const uint16_t* x, int batch, int k, int chunk, int kch);
// Enqueue the chunk selection.  pdl: launched with programmatic serialization
// (it may start while the previous kernel drains; it releases its dependents at
// its start, so a following kernel launched the same way can overlap its
// selection-independent prologue with it).
sf_status launch_select(const uint16_t* x, int batch, int k, int chunk, int kch, int32_t* sel,
                        cudaStream_t s, bool pdl);

}  // namespace sf
