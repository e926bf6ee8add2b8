// plan.h -- host-side planning of a Muon step: orientation, padded strides and
// the tile lists walked by the persistent tensor-core GEMMs.  Plain C++, no CUDA.
#pragma once

#include <cstdint>
#include <vector>

namespace muon {

struct GroupDims {
    int rows, cols, count;
    int m, n;          // oriented: m = min(rows, cols), n = max(rows, cols)
    int ldm, ldn;      // strides rounded up to 8 elements (16 bytes of bf16)
    int transposed;    // rows > cols ("Muon" section 4: transpose to the smaller Gram)
};

struct Tile { int group, mat, tile_row, tile_col; };

inline int round_up8(int x) { return (x + 7) & ~7; }

GroupDims make_dims(int rows, int cols, int count);

// phase 0 = GRAM (K = n), 1 = POLY (K = m), 2 = UPDATE (K = m).
// GRAM / POLY: tiles of the m x m output that hold at least one element with col >= row.
// UPDATE: every tile of the m x n output.  Sorted by K (the per-tile cost)
// descending, ties in (group, matrix, tile_row, tile_col) order.
std::vector<Tile> build_tiles(const std::vector<GroupDims>& groups, int phase, int bm, int bn);

// 1 unless the environment variable MUON_GEMM_PAIR is "0" (see kernels.cuh).
int tc_gemm_default_pair();

}  // namespace muon
