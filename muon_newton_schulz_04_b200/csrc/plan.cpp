// plan.cpp -- tile lists of the grouped persistent GEMMs (see plan.h).
#include "plan.h"

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <map>
#include <tuple>

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

int active_clusters(const UnitPlan& up, int clusters) {
    if ((int)up.begin.size() < clusters + 1) return clusters;
    int k = 0;
    while (k < clusters && up.begin[k + 1] > up.begin[k]) ++k;
    for (int c = k; c < clusters; ++c)
        if (up.begin[c + 1] > up.begin[c]) return clusters;
    return k;
}

std::string check_plan(const std::vector<GroupDims>& groups, int phase, int bm, int bn, int bk,
                       const std::vector<Tile>& tiles, const std::vector<int>& kblocks, const UnitPlan* up,
                       int clusters) {
    using Key = std::tuple<int, int, int, int>;
    auto msg = [](const char* what, long long i) { return std::string(what) + " (entry " + std::to_string(i) + ")"; };
    if (kblocks.size() != tiles.size()) return "one K-block count per tile expected";
    long long expected = 0;
    for (const GroupDims& d : groups) {
        const int out_cols = (phase == 2) ? d.n : d.m;
        const long long tr = (d.m + bm - 1) / bm, tc = (out_cols + bn - 1) / bn;
        long long per = 0;
        for (long long i = 0; i < tr; ++i)
            for (long long j = 0; j < tc; ++j)
                if (phase == 2 || std::min((j + 1) * bn, (long long)d.m) - 1 >= i * bm) ++per;
        expected += per * d.count;
    }
    if ((long long)tiles.size() != expected) return "tile count differs from the shapes' tile count";
    std::map<Key, int> index;
    for (size_t i = 0; i < tiles.size(); ++i) {
        const Tile& t = tiles[i];
        if (t.group < 0 || t.group >= (int)groups.size()) return msg("tile group out of range", i);
        const GroupDims& d = groups[t.group];
        const int out_cols = (phase == 2) ? d.n : d.m;
        if (t.mat < 0 || t.mat >= d.count) return msg("tile matrix out of range", i);
        if (t.tile_row < 0 || (long long)t.tile_row * bm >= d.m) return msg("tile row out of range", i);
        if (t.tile_col < 0 || (long long)t.tile_col * bn >= out_cols) return msg("tile column out of range", i);
        if (phase != 2 && std::min((long long)(t.tile_col + 1) * bn, (long long)d.m) - 1 < (long long)t.tile_row * bm)
            return msg("symmetric tile entirely below the diagonal", i);
        const int k = (phase == 0) ? d.n : d.m;
        if (kblocks[i] != (k + bk - 1) / bk) return msg("wrong K-block count", i);
        if (!index.emplace(Key{t.group, t.mat, t.tile_row, t.tile_col}, (int)i).second) return msg("duplicate tile", i);
    }
    if (up == nullptr) return "";
    const std::vector<Unit>& us = up->units;
    if ((int)up->begin.size() != clusters + 1 || up->begin.front() != 0 || up->begin.back() != (int)us.size())
        return "cluster offsets do not span the unit list";
    for (int c = 0; c < clusters; ++c)
        if (up->begin[c] > up->begin[c + 1]) return msg("cluster offsets decrease", c);
    std::vector<std::vector<int>> of(tiles.size());
    for (size_t i = 0; i < us.size(); ++i) {
        const Unit& u = us[i];
        auto it = index.find(Key{u.tile.group, u.tile.mat, u.tile.tile_row, u.tile.tile_col});
        if (it == index.end()) return msg("unit of a tile not in the list", i);
        const int kb = kblocks[it->second];
        if (u.k_begin < 0 || u.k_begin >= u.k_end || u.k_end > kb) return msg("unit K range outside its tile", i);
        if (u.kind < 0 || u.kind > 2 || u.n_half < 0 || u.n_half > 2) return msg("unit kind or half out of range", i);
        if (u.n_half != 0 && (u.kind != 0 || u.k_begin != 0 || u.k_end != kb)) return msg("column half is not a whole-K unit", i);
        if (u.kind == 1 && (u.k_begin != 0 || u.nslots < 1)) return msg("split head does not start at K-block 0", i);
        if (u.kind != 0 && (u.slot < 0 || u.slot + (u.kind == 1 ? u.nslots : 1) > up->nslots))
            return msg("partial-sum slot out of range", i);
        of[it->second].push_back((int)i);
    }
    for (size_t t = 0; t < tiles.size(); ++t) {
        std::vector<int> l = of[t];
        const int kb = kblocks[t];
        if (l.empty()) return msg("tile without a unit", t);
        if (l.size() == 1) {
            const Unit& u = us[l[0]];
            if (u.kind != 0 || u.n_half != 0 || u.k_begin != 0 || u.k_end != kb) return msg("single unit is not the whole tile", t);
            continue;
        }
        if (us[l[0]].n_half != 0) {
            if (l.size() != 2 || us[l[0]].n_half + us[l[1]].n_half != 3 || us[l[1]].n_half == 0)
                return msg("column halves do not pair up", t);
            continue;
        }
        std::sort(l.begin(), l.end(), [&](int a, int b) { return us[a].k_begin < us[b].k_begin; });
        const Unit& head = us[l[0]];
        if (head.kind != 1 || head.nslots != (int)l.size() - 1) return msg("split tile without a matching head", t);
        for (size_t i = 1; i < l.size(); ++i) {
            const Unit& u = us[l[i]];
            if (u.kind != 2 || u.n_half != 0) return msg("split part of the wrong kind", t);
            if (u.k_begin != us[l[i - 1]].k_end) return msg("split parts leave a gap or overlap", t);
            if (u.slot != head.slot + (int)i - 1) return msg("split part slot out of order", t);
        }
        if (us[l.back()].k_end != kb) return msg("split parts stop before the last K-block", t);
    }
    return "";
}

int tc_gemm_split_tiles() {
    const char* v = std::getenv("MUON_GEMM_SPLIT");
    return (v && std::strcmp(v, "1") == 0) ? 1 : 0;
}

int tc_gemm_fused_apply() {
    const char* v = std::getenv("MUON_FUSED_APPLY");
    return (v && std::strcmp(v, "1") == 0) ? 1 : 0;
}

int tc_gemm_default_pair() {
    const char* v = std::getenv("MUON_GEMM_PAIR");
    return (v && std::strcmp(v, "0") == 0) ? 0 : 1;
}

}  // namespace muon
