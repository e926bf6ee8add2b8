// plan.cpp -- tile lists of the grouped persistent GEMMs (see plan.h).
#include "plan.h"

#include <algorithm>
#include <cstdlib>
#include <cstring>

namespace muon {

GroupDims make_dims(int rows, int cols, int count) {
    GroupDims d{};
    d.rows = rows;
    d.cols = cols;
    d.count = count;
    d.transposed = rows > cols ? 1 : 0;
    d.m = rows > cols ? cols : rows;
    d.n = rows > cols ? rows : cols;
    d.ldm = round_up8(d.m);
    d.ldn = round_up8(d.n);
    return d;
}

std::vector<Tile> build_tiles(const std::vector<GroupDims>& groups, int phase, int bm, int bn) {
    std::vector<Tile> tiles;
    std::vector<int> cost;
    for (int g = 0; g < (int)groups.size(); ++g) {
        const GroupDims& d = groups[g];
        const int out_cols = (phase == 2) ? d.n : d.m;
        const int tr = (d.m + bm - 1) / bm;
        const int tc = (out_cols + bn - 1) / bn;
        const int k = (phase == 0) ? d.n : d.m;
        for (int z = 0; z < d.count; ++z) {
            for (int i = 0; i < tr; ++i) {
                for (int j = 0; j < tc; ++j) {
                    if (phase != 2) {
                        // keep the tile if its last column reaches its first row
                        const long long last_col = std::min((long long)(j + 1) * bn, (long long)d.m) - 1;
                        if (last_col < (long long)i * bm) continue;
                    }
                    tiles.push_back(Tile{g, z, i, j});
                    cost.push_back(k);
                }
            }
        }
    }
    std::vector<int> order(tiles.size());
    for (size_t i = 0; i < order.size(); ++i) order[i] = (int)i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
    std::vector<Tile> out;
    out.reserve(tiles.size());
    for (int i : order) out.push_back(tiles[i]);
    return out;
}

int tc_gemm_default_pair() {
    const char* v = std::getenv("MUON_GEMM_PAIR");
    return (v && std::strcmp(v, "0") == 0) ? 0 : 1;
}

}  // namespace muon
