// Host-side test of muon::check_plan (built and run by test_plan_check_cpu.py):
// every plan the planner builds passes, and each planted defect is reported.
#include <cstdio>
#include <string>
#include <vector>

#include "plan.h"

using namespace muon;

static int failures = 0;

static void expect(bool ok, const char* what) {
    if (!ok) {
        std::printf("FAIL: %s\n", what);
        ++failures;
    }
}

struct Case {
    std::vector<GroupDims> dims;
    std::vector<Tile> tiles;
    std::vector<int> kb;
    UnitPlan up;
};

static Case make(const std::vector<std::vector<int>>& shapes, int phase, int clusters, bool split) {
    Case c;
    for (const auto& s : shapes) c.dims.push_back(make_dims(s[0], s[1], s[2]));
    c.tiles = build_tiles(c.dims, phase, 256, 256);
    for (const Tile& t : c.tiles) c.kb.push_back(((phase == 0 ? c.dims[t.group].n : c.dims[t.group].m) + 63) / 64);
    c.up = build_units(c.tiles, c.kb, clusters, split, !split);
    return c;
}

static std::string check(const Case& c, int phase, int clusters) {
    return check_plan(c.dims, phase, 256, 256, 64, c.tiles, c.kb, &c.up, clusters);
}

int main() {
    const std::vector<std::vector<std::vector<int>>> sets = {
        {{4096, 4096, 1}}, {{768, 768, 48}, {3072, 768, 12}, {768, 3072, 12}}, {{1000, 37, 1}, {37, 1000, 2}},
        {{2048, 2560, 1}}, {{3328, 3328, 1}}, {{1, 1, 3}, {64, 1, 1}, {300, 129, 2}}, {{1600, 1600, 8}, {6400, 1600, 2}}};
    for (const auto& shapes : sets)
        for (int phase = 0; phase < 3; ++phase)
            for (int clusters : {1, 7, 74})
                for (bool split : {false, true}) {
                    Case c = make(shapes, phase, clusters, split);
                    const std::string r = check(c, phase, clusters);
                    if (!r.empty()) std::printf("valid plan rejected: %s\n", r.c_str());
                    expect(r.empty(), "planner output passes");
                    expect(check_plan(c.dims, phase, 256, 256, 64, c.tiles, c.kb, nullptr, clusters).empty(),
                           "tile list alone passes");
                }
    // the one-CTA kernel's 128 x 256 tiles (tile list only: it walks tiles, not units)
    for (const auto& shapes : sets)
        for (int phase = 0; phase < 3; ++phase) {
            std::vector<GroupDims> dims;
            for (const auto& sh : shapes) dims.push_back(make_dims(sh[0], sh[1], sh[2]));
            const std::vector<Tile> tiles = build_tiles(dims, phase, 128, 256);
            std::vector<int> kb;
            for (const Tile& t : tiles) kb.push_back(((phase == 0 ? dims[t.group].n : dims[t.group].m) + 63) / 64);
            expect(check_plan(dims, phase, 128, 256, 64, tiles, kb, nullptr, 1).empty(), "128 x 256 tile list passes");
        }
    // planted defects, each on a fresh copy of a valid plan
    const std::vector<std::vector<int>> shapes = {{768, 768, 4}, {3072, 768, 2}, {520, 264, 1}};
    for (int phase = 0; phase < 3; ++phase) {
        const int C = 5;
        Case base = make(shapes, phase, C, true);
        expect(check(base, phase, C).empty(), "split base plan passes");
        { Case c = base; c.tiles.pop_back(); c.kb.pop_back(); expect(!check(c, phase, C).empty(), "missing tile"); }
        { Case c = base; c.tiles[1] = c.tiles[0]; expect(!check(c, phase, C).empty(), "duplicate tile"); }
        { Case c = base; c.tiles[0].tile_row += 50; expect(!check(c, phase, C).empty(), "tile row out of range"); }
        { Case c = base; c.tiles[0].mat = 9; expect(!check(c, phase, C).empty(), "matrix out of range"); }
        if (phase != 2) {
            // a tile strictly below the diagonal of a 768 x 768 matrix (3 x 3 tiles)
            Case c = base;
            for (Tile& t : c.tiles)
                if (t.group == 0 && t.tile_row == 0 && t.tile_col == 0) { t.tile_row = 2; break; }
            expect(!check(c, phase, C).empty(), "symmetric tile below the diagonal");
        }
        { Case c = base; c.kb[0] += 1; expect(!check(c, phase, C).empty(), "wrong K-block count"); }
        { Case c = base; c.up.units[0].k_end -= 1; expect(!check(c, phase, C).empty(), "short unit"); }
        { Case c = base; c.up.units.pop_back(); c.up.begin.back() -= 1; expect(!check(c, phase, C).empty(), "dropped unit"); }
        { Case c = base; c.up.begin[1] = c.up.begin[2] + 1; expect(!check(c, phase, C).empty(), "offsets decrease"); }
        { Case c = base; c.up.units[0].kind = 3; expect(!check(c, phase, C).empty(), "bad kind"); }
        {
            Case c = base;
            bool planted = false;
            for (Unit& u : c.up.units)
                if (u.kind == 2) { u.slot += 1; planted = true; break; }
            if (planted) expect(!check(c, phase, C).empty(), "split part slot");
            planted = false;
            for (Unit& u : c.up.units)
                if (u.kind == 2) { u.k_begin += 1; planted = u.k_begin < u.k_end; break; }
            if (planted) expect(!check(c, phase, C).empty(), "gap between split parts");
        }
        // a plan with column halves: 4 tiles on 3 clusters leave 1 tile, cut in two
        Case h = make({{1024, 256, 1}}, 2, 3, false);
        expect(check(h, 2, 3).empty(), "half plan passes");
        bool halves = false;
        for (const Unit& u : h.up.units) halves = halves || u.n_half != 0;
        expect(halves, "half plan has column halves");
        for (Unit& u : h.up.units)
            if (u.n_half == 2) { u.n_half = 1; break; }
        expect(!check(h, 2, 3).empty(), "halves that do not pair up");
    }
    // clusters launched: the busy ones form a prefix of the deal
    {
        Case few = make({{256, 512, 1}}, 2, 74, false);           // 2 update tiles on 74 clusters
        expect(active_clusters(few.up, 74) == 2, "two tiles keep two clusters busy");
        Case full = make({{4096, 4096, 1}}, 2, 74, false);        // 256 tiles: every cluster
        expect(active_clusters(full.up, 74) == 74, "a full plan keeps every cluster");
        Case half = make({{1024, 256, 1}}, 2, 3, false);           // 3 whole tiles + 2 halves on 3 clusters
        expect(active_clusters(half.up, 3) == 3, "halves keep their clusters");
        Case gap = few;                                            // work moved behind an idle cluster
        gap.up.begin = std::vector<int>(75, 2);
        gap.up.begin[0] = 0; gap.up.begin[1] = 1; gap.up.begin[2] = 1;
        for (int c = 3; c <= 74; ++c) gap.up.begin[c] = 2;
        expect(active_clusters(gap.up, 74) == 74, "busy clusters that are not a prefix launch all");
        UnitPlan none;
        none.begin = std::vector<int>(75, 0);
        expect(active_clusters(none, 74) == 0, "no work, no cluster");
    }
    std::printf(failures == 0 ? "plan check ok\n" : "plan check: %d failures\n", failures);
    return failures == 0 ? 0 : 1;
}
