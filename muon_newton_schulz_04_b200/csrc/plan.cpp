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

UnitPlan build_units(const std::vector<Tile>& tiles, const std::vector<int>& kblocks, int clusters, bool split,
                     bool half_tail) {
    UnitPlan up;
    const int T = (int)tiles.size();
    const int C = clusters < 1 ? 1 : clusters;
    const int rem = T % C;
    const bool halves = !split && half_tail && rem > 0 && T >= C && 2 * rem <= C;
    const int R = (split || halves) ? rem : 0;
    const int D = T - R;
    std::vector<std::vector<Unit>> per(C);
    for (int t = 0; t < D; ++t) per[t % C].push_back(Unit{tiles[t], 0, kblocks[t], 0, 0, 0, 0});
    if (halves) {
        for (int r = 0; r < R; ++r)
            for (int h = 0; h < 2; ++h) per[2 * r + h].push_back(Unit{tiles[D + r], 0, kblocks[D + r], 0, 0, 0, 1 + h});
        up.begin.push_back(0);
        for (int c = 0; c < C; ++c) {
            up.units.insert(up.units.end(), per[c].begin(), per[c].end());
            up.begin.push_back((int)up.units.size());
        }
        return up;
    }
    if (R > 0) {
        // flatten the remaining tiles' K-blocks and cut them into C ranges
        long long total = 0;
        std::vector<long long> start(R + 1, 0);
        for (int r = 0; r < R; ++r) { start[r] = total; total += kblocks[D + r]; }
        start[R] = total;
        std::vector<std::vector<Unit>> sk(C);
        std::vector<std::vector<int>> tile_units(R);     // (cluster) of each part, in K order
        std::vector<std::vector<int>> tile_pos(R);
        for (int c = 0; c < C; ++c) {
            long long a = total * c / C, b = total * (c + 1) / C;
            int r = 0;
            while (r < R && start[r + 1] <= a) ++r;
            while (a < b && r < R) {
                const long long e = std::min(b, start[r + 1]);
                const int kb = (int)(a - start[r]), ke = (int)(e - start[r]);
                tile_units[r].push_back(c);
                tile_pos[r].push_back((int)sk[c].size());
                sk[c].push_back(Unit{tiles[D + r], kb, ke, kb == 0 ? 1 : 2, 0, 0, 0});
                a = e;
                ++r;
            }
        }
        int slot = 0;
        for (int r = 0; r < R; ++r) {
            const int n = (int)tile_units[r].size();
            if (n == 1) { sk[tile_units[r][0]][tile_pos[r][0]].kind = 0; continue; }
            Unit& head = sk[tile_units[r][0]][tile_pos[r][0]];
            head.kind = 1;
            head.slot = slot;
            head.nslots = n - 1;
            for (int i = 1; i < n; ++i) {
                Unit& part = sk[tile_units[r][i]][tile_pos[r][i]];
                part.kind = 2;
                part.slot = slot++;
            }
        }
        up.nslots = slot;
        for (int c = 0; c < C; ++c) per[c].insert(per[c].end(), sk[c].begin(), sk[c].end());
    }
    up.begin.push_back(0);
    for (int c = 0; c < C; ++c) {
        up.units.insert(up.units.end(), per[c].begin(), per[c].end());
        up.begin.push_back((int)up.units.size());
    }
    return up;
}

int tc_gemm_split_tiles() {
    const char* v = std::getenv("MUON_GEMM_SPLIT");
    return (v && std::strcmp(v, "1") == 0) ? 1 : 0;
}

int tc_gemm_default_pair() {
    const char* v = std::getenv("MUON_GEMM_PAIR");
    return (v && std::strcmp(v, "0") == 0) ? 0 : 1;
}

}  // namespace muon
