// Where row r of a row buffer lives, for the kernels that move whole rows: one buffer on
// this GPU (Local*), or, for expert parallelism across GPUs, rank r / C's buffer at local
// row r % C through the pointer this process has for it -- its own buffer, or a peer GPU's
// mapped into this process (Rank*).  The rank tables are kernel parameters
// (__grid_constant__), one entry per rank.
#pragma once
#include "common.cuh"

namespace moe {

struct LocalY {  // rows read
  const uint4* base;
  __device__ __forceinline__ const uint4* row(int64_t r, int dv) const { return base + r * dv; }
};
struct RankY {
  const uint4* base[MOE_EP_MAX_RANKS];
  int C;
  __device__ __forceinline__ const uint4* row(int64_t r, int dv) const {
    const int ri = (int)r;  // rows of the job < 2^31
    const int u = ri / C;
    return base[u] + (int64_t)(ri - u * C) * dv;
  }
};
struct LocalRows {  // rows written
  uint4* base;
  __device__ __forceinline__ uint4* row(int64_t r, int dv) const { return base + r * dv; }
};
struct RankRows {
  uint4* base[MOE_EP_MAX_RANKS];
  int C;
  __device__ __forceinline__ uint4* row(int64_t r, int dv) const {
    const int ri = (int)r;  // rows of the job < 2^31
    const int u = ri / C;
    return base[u] + (int64_t)(ri - u * C) * dv;
  }
};

}  // namespace moe
