// fa_bwd.cuh — exact attention backward for sm_100a.
#pragma once
#include "sm100.cuh"

namespace fa {

// Workspace: fp32 dQ accumulator [rows, d] followed by the fp32 row term D [rows].
inline size_t bwd_workspace_bytes(size_t rows, int d) {
  return rows * static_cast<size_t>(d) * 4 + ((rows * 4 + 255) / 256) * 256;
}

}  // namespace fa
