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
  unsigned long long* counters;  // [R][2] arrival counters (counter_arrive)
  unsigned long long gen;        // this call's counter generation
};

// Up to kInlineGroups groups travel with the launch itself, as a kernel parameter (the
// TMA descriptors then sit in parameter space, where a launch's tensor maps normally live),
// so a call with few groups needs no host-to-device copy of its table.
constexpr int kInlineGroups = 16;
struct GroupTableInline {
  GroupDesc d[kInlineGroups];
};

// Writes G records to dst (device, 64-byte aligned) on `stream` through kernels whose
// parameters carry the records (no host-memory copy: graph-capturable).
cudaError_t launch_upload_group_table(const GroupDesc* table, int G, GroupDesc* dst, cudaStream_t stream);

// `inl` (nullable): the table as a kernel parameter (G <= kInlineGroups); else p.groups.
cudaError_t launch_gemm_grouped_split(const GroupedParams& p, const GroupedSplit& sp, const GroupTableInline* inl,
                                      int clusters, cudaStream_t stream);

}  // namespace smg
