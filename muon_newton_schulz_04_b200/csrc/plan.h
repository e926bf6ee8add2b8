// plan.h -- host-side planning of a Muon step: orientation, padded strides and
// the tile lists walked by the persistent tensor-core GEMMs.  Plain C++, no CUDA.
#pragma once

#include <cstdint>
#include <string>
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

// Work units of the persistent two-CTA kernel.  Each unit is a tile and a K-block
// range [k_begin, k_end) of it:
//   kind 0: the whole tile, finished by its unit;
//   kind 1: the head of a split tile (k_begin = 0): adds the fp32 partial sums of
//           slots [slot, slot + nslots) after its own range, then finishes the tile;
//   kind 2: a later part of a split tile: writes its fp32 partial sum to `slot`.
// Units are listed per cluster in execution order; cluster c runs
// units[begin[c] .. begin[c+1]).  The tiles of full rounds (floor(T / C) * C of them,
// T tiles, C clusters) are whole units dealt round-robin; when split is true and
// T % C != 0, the K-blocks of the remaining tiles are divided into C contiguous,
// nearly equal ranges, one per cluster, so every cluster ends at about the same
// time.  A cluster's range starts with at most one kind-2 unit, so a head unit only
// waits for partials that their clusters produce before doing anything else.
//   n_half: 0 = all 256 columns of the tile; 1 / 2 = its first / second 128 columns
//           (an independent output block with the full K range).
struct Unit { Tile tile; int k_begin, k_end, kind, slot, nslots, n_half; };

struct UnitPlan {
    std::vector<Unit> units;
    std::vector<int> begin;   // C + 1 offsets
    int nslots = 0;           // partial-sum slots used
};

// half_tail: when split is false and the R = T % C remaining tiles fit as 2R halves
// on the C clusters (2R <= C), they are cut along N into two 128-column halves,
// one per cluster, so the last round takes about half as long.
UnitPlan build_units(const std::vector<Tile>& tiles, const std::vector<int>& kblocks, int clusters, bool split,
                     bool half_tail = false);

// Clusters of a unit plan that have work.  build_units deals from cluster 0, so they
// are a prefix; a phase with fewer units than clusters then launches only those and
// the idle clusters skip their set-up (TMEM allocation, barriers, cluster sync).
// Returns `clusters` when the busy clusters are not a prefix (every cluster is
// launched), 0 when no cluster has work.
int active_clusters(const UnitPlan& up, int clusters);

// Host-side check of a plan before anything is launched with it: the tile list of
// `phase` holds every tile it should exactly once (in range, and for GRAM / POLY
// touching col >= row), kblocks[i] is tile i's K-block count, and -- when `up` is
// given -- the units of `clusters` clusters cover each tile exactly once: one whole
// unit, two column halves, or a head (kind 1, from K-block 0) and kind-2 parts that
// continue its K range without gaps, with consistent partial-sum slots.  Returns an
// empty string when the plan is valid, else what is wrong.
std::string check_plan(const std::vector<GroupDims>& groups, int phase, int bm, int bn, int bk,
                       const std::vector<Tile>& tiles, const std::vector<int>& kblocks, const UnitPlan* up,
                       int clusters);

// 0 unless the environment variable MUON_GEMM_SPLIT is "1": split the K-blocks of
// the last, partial round of tiles over all clusters (build_units).  Off by
// default: on the 4096 x 4096 workload it measured slower than whole tiles.
int tc_gemm_split_tiles();

// 0 unless the environment variable MUON_FUSED_APPLY is "1".  With 1 the bf16 path
// applies W <- decay*W - lr*s*O (or copies O out) in the epilogue of the last update
// GEMM; by default the update GEMM only writes O and the apply kernel does the rest.
// The fused form moves 4 B/elem less but measured slower on the GPT-2 and 4096^2
// workloads (its epilogue warps, one matrix row per lane, wait on W's reads while the
// accumulator they hold stalls the MMAs) and within noise on the MoE one.
int tc_gemm_fused_apply();

// 1 unless the environment variable MUON_GEMM_PAIR is "0" (see kernels.cuh).
int tc_gemm_default_pair();

}  // namespace muon
