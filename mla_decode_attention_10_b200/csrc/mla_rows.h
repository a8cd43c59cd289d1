// mla_rows.h -- the large-batch (MLA_MODE_ROWS) kernel of the epilogue:
// plan and kernel lookup for the launcher in mla_epilogue.cu (internal).
#pragma once

#include <cstddef>
#include <cstdint>

#include "mla_epilogue.h"

namespace mla {

// Upper limits (and defaults) of the tuning knobs mla_epilogue_set_tuning
// clamps to.
constexpr int kRowsMaxBlocksPerSm = 1;     // persistent: one block per SM (184 KB of shared memory)
constexpr int kRowsMaxConsumerWarps = 16;  // consumer warps beside the producer warp
constexpr int kRowsDefaultWarps = 8;

// Grid and block of a ROWS launch over `rows` rows.
void rows_plan(int64_t rows, bool qf8, bool kvf8, int32_t sm_count, int32_t blocks_per_sm, int32_t warps_per_block,
               mla_plan* p);

// The ROWS kernel for flags & 7 and its dynamic shared memory; makes the
// kernel's shared-memory opt-in on device `dev` the first time.
mla_status rows_kernel(int flag_bits, int dev, const void** fn, size_t* smem_bytes);

}  // namespace mla
