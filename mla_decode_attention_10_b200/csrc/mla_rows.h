// mla_rows.h -- the large-batch (MLA_MODE_ROWS) kernel of the epilogue:
// plan and kernel lookup for the launcher in mla_epilogue.cu (internal).
#pragma once

#include <cstddef>
#include <cstdint>

#include "mla_epilogue.h"

namespace mla {

// Upper limits (and defaults) of the tuning knobs mla_epilogue_set_tuning
// clamps to.
constexpr int kRowsMaxBlocksPerSm = 5;  // resident blocks per SM the kernels are compiled for, at most
constexpr int kRowsMaxWarps = 8;        // warps per block
constexpr int kRowsDefaultWarps = 8;

// Grid and block of a ROWS launch over `rows` rows.
void rows_plan(int64_t rows, bool qf8, bool kvf8, int32_t sm_count, int32_t blocks_per_sm, int32_t warps_per_block,
               mla_plan* p);

// The ROWS kernel for flags & 7 and its dynamic shared memory for blocks of
// `warps` warps.
mla_status rows_kernel(int flag_bits, int warps, const void** fn, size_t* smem_bytes);

}  // namespace mla
