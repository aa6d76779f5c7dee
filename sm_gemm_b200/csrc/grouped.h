// Grouped GEMM: the split of a ragged last wave (gemm_grouped.cu). The last R tiles of
// the launch's tile order are split along K into S pieces; piece u of tail tile r = u / S
// writes its partial to slots[u][rank] and the last piece of the tile to arrive sums them.
#pragma once

#include "kernels.h"

namespace smg {

struct GroupedSplit {
  long long split_tiles;    // R (0: no split)
  int splits;               // S pieces per split tile
  float* slots;             // [R * S][2 ranks][128][256] float partials
  int* counters;            // [R][2], zeroed before the launch
};

cudaError_t launch_gemm_grouped_split(const GroupedParams& p, const GroupedSplit& sp, int clusters,
                                      cudaStream_t stream);

}  // namespace smg
