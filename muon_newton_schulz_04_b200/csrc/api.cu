// api.cu -- the C ABI of include/muon.h: validation, the per-shape plan cache,
// the library-owned workspace, TMA descriptors and the launch sequence of one
// Muon step ("Muon: An optimizer for hidden layers in neural networks",
// section 4):
//
//   momentum_norm  ->  ns_steps x (GRAM -> POLY -> UPDATE)  ->  apply
//   (with MUON_FUSED_APPLY=1 the bf16 path's last UPDATE applies W in its epilogue
//   and no apply kernel runs)
//
// All launches go to the caller's stream; nothing here synchronises except the
// entry points documented to do so.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <functional>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/muon.h"
#include "kernels.cuh"
#include "plan.h"

using namespace muon;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct DevBuf {
    void* ptr = nullptr;
    size_t size = 0;
};

// Workspace offsets of one group (bytes from the workspace base).
struct GroupOffsets {
    size_t xb[2], xl, xf[2], a, p;
};

struct Plan {
    std::vector<int> key;                // (rows, cols, count) per group + precision
    std::vector<GroupDims> dims;
    std::vector<GroupOffsets> offs;
    std::vector<int> mat_base;           // global matrix index of each group's first matrix
    int nmat = 0;
    int k1_blocks = 0, k7_blocks = 0;
    std::vector<EwSeg> segs;             // shape part filled at plan time
    // tile lists (tensor-core path)
    int n_gram = 0, n_poly = 0, n_upd = 0;
    int var[3] = {1, 0, 0};              // two-CTA shared-memory configuration per phase
    bool fused_apply = false;            // bf16 path: the last update also applies W (else the apply kernel)
    // device addresses inside the workspace
    int4* d_tiles_gram = nullptr; int4* d_tiles_poly = nullptr; int4* d_tiles_upd = nullptr;
    // two-CTA kernel: per-phase unit lists (plan.h) and the split-tile partial sums
    int4* d_units[3] = {nullptr, nullptr, nullptr};
    int* d_unit_begin[3] = {nullptr, nullptr, nullptr};
    int unit_clusters = 0;
    int active[3] = {0, 0, 0};           // per phase: clusters that have units (launched)
    float* d_sk_partial = nullptr;
    int* d_sk_count = nullptr;
    int* d_sk_flag = nullptr;
    GemmMaps* d_maps = nullptr;
    GemmGroupInfo* d_ginfo = nullptr;
    EwSeg* d_segs = nullptr;
    double* d_partials = nullptr;
    float* d_norms = nullptr;
    float* d_scale = nullptr;
    int* d_counters = nullptr;           // per-matrix block counters of the momentum kernel
    double* d_rms_part = nullptr;        // update-RMS partial sums (UPDATE_RMS_PARTIALS per matrix)
    float* d_rms = nullptr;              // update RMS per matrix
    bool valid = false;
    unsigned long long version = 0;      // distinct per built plan
    std::vector<EwSeg> uploaded;         // last segment table copied to the device
};

}  // namespace

struct muon_handle {
    muon_config cfg;
    int device = 0;
    int num_sms = 148;
    int pair = 1;            // 1: two-CTA GEMM kernel, 0: one-CTA kernel
    int max_clusters = 74;   // co-resident two-CTA clusters of the pair kernel
    std::string last_error;
    DevBuf ws;            // plan workspace
    DevBuf staging;       // muon_step_host staging
    DevBuf scratch;       // muon_ns_phase_run descriptors
    size_t mem_limit = 0;  // cap on ws + staging + scratch (0: none), muon_set_memory_limit
    int* d_err = nullptr;
    Plan plan;
    EncodeTiledFn encode = nullptr;
    int epoch = 0;           // distinct per two-CTA GEMM launch (split-tile flags)
    bool tc_ready = false;
    // per-phase timing
    bool timing = false;
    std::vector<cudaEvent_t> ev_free;
    struct Pending { int kind; cudaEvent_t a, b; };
    std::vector<Pending> pending;
    double t_ms[MUON_TIMING_KINDS] = {};
    int t_n[MUON_TIMING_KINDS] = {};
    // muon_step_host: side streams for copies that overlap the GEMMs (W up, B down),
    // and their events
    cudaStream_t side = nullptr, side2 = nullptr;
    // captured launch sequence of muon_step / muon_orthogonalize (replayed while the
    // plan, the caller's pointers and the configuration stay the same)
    bool graphs = true;
    cudaStream_t cap_stream = nullptr;
    cudaGraphExec_t gexec = nullptr;
    std::vector<EwSeg> g_segs;
    muon_config g_cfg;
    void* g_ws = nullptr;
    int g_mode = -1;
    unsigned long long g_version = 0;
    unsigned long long plans_built = 0;
    cudaEvent_t ev_start = nullptr, ev_w = nullptr, ev_k1 = nullptr, ev_done = nullptr;
    // muon_apply: segment table of the last call (device copy in apply_segs)
    DevBuf apply_segs;
    std::vector<EwSeg> apply_uploaded;
};

namespace {

muon_status fail(muon_handle* h, muon_status s, const char* fmt, ...) {
    if (h) {
        char buf[512];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof(buf), fmt, ap);
        va_end(ap);
        h->last_error = buf;
    }
    return s;
}

#define CUDA_TRY(h, expr)                                                                          \
    do {                                                                                           \
        cudaError_t e_ = (expr);                                                                   \
        if (e_ != cudaSuccess)                                                                     \
            return fail((h), MUON_ERR_CUDA, "%s failed: %s (%s:%d)", #expr, cudaGetErrorString(e_), \
                        __FILE__, __LINE__);                                                       \
    } while (0)

struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) cudaSetDevice(dev);
        else prev = -1;
    }
    ~DeviceGuard() { if (prev >= 0) cudaSetDevice(prev); }
};

bool finite(float x) { return std::isfinite(x); }

cudaEvent_t take_event(muon_handle* h) {
    if (!h->ev_free.empty()) {
        cudaEvent_t e = h->ev_free.back();
        h->ev_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) { cudaGetLastError(); return nullptr; }
    return e;
}

// Brackets one launch with events when timing is on.
struct PhaseTimer {
    muon_handle* h;
    int kind;
    cudaStream_t s;
    cudaEvent_t a = nullptr;
    PhaseTimer(muon_handle* h_, int kind_, cudaStream_t s_) : h(h_), kind(kind_), s(s_) {
        if (h->timing && (a = take_event(h)) != nullptr) cudaEventRecord(a, s);
    }
    void done() {
        if (!a) return;
        cudaEvent_t b = take_event(h);
        if (!b) { h->ev_free.push_back(a); a = nullptr; return; }
        cudaEventRecord(b, s);
        h->pending.push_back(muon_handle::Pending{kind, a, b});
        a = nullptr;
    }
};

// Host-side NVTX range (a no-op unless a profiler is attached): one per entry
// point and one per enqueued phase, named like the timing kinds.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
const char* const kPhaseNames[MUON_TIMING_KINDS] = {"momentum_norm", "norm_finalize", "gram", "poly", "update", "apply"};

#define TIMED(h, kind, s, expr)                \
    do {                                       \
        NvtxRange nr_(kPhaseNames[(kind)]);    \
        PhaseTimer pt_((h), (kind), (s));      \
        CUDA_TRY((h), (expr));                 \
        pt_.done();                            \
    } while (0)

muon_status check_config(const muon_config* c, std::string* why) {
    if (!c) { *why = "config is NULL"; return MUON_ERR_INVALID; }
    if (!finite(c->lr)) { *why = "lr is not finite"; return MUON_ERR_INVALID; }
    if (!(c->momentum >= 0.f && c->momentum < 1.f)) { *why = "momentum must be in [0, 1)"; return MUON_ERR_INVALID; }
    if (!(finite(c->weight_decay) && c->weight_decay >= 0.f)) { *why = "weight_decay must be finite and >= 0"; return MUON_ERR_INVALID; }
    if (!(finite(c->eps) && c->eps >= 0.f)) { *why = "eps must be finite and >= 0"; return MUON_ERR_INVALID; }
    if (c->nesterov != 0 && c->nesterov != 1) { *why = "nesterov must be 0 or 1"; return MUON_ERR_INVALID; }
    if (c->ns_steps < 0 || c->ns_steps > 16) { *why = "ns_steps must be in [0, 16]"; return MUON_ERR_INVALID; }
    if (!(finite(c->ns_a) && finite(c->ns_b) && finite(c->ns_c))) { *why = "ns coefficients must be finite"; return MUON_ERR_INVALID; }
    if (c->scale_mode < MUON_SCALE_NONE || c->scale_mode > MUON_SCALE_CUSTOM) { *why = "bad scale_mode"; return MUON_ERR_INVALID; }
    if (c->scale_mode == MUON_SCALE_MATCH_RMS && !(finite(c->rms_target) && c->rms_target > 0.f)) { *why = "rms_target must be finite and > 0"; return MUON_ERR_INVALID; }
    if (c->precision != MUON_PREC_BF16 && c->precision != MUON_PREC_FP32_DEBUG) { *why = "bad precision"; return MUON_ERR_INVALID; }
    return MUON_OK;
}

// Common shape checks of one group of `count` rows x cols matrices.
muon_status check_shape(int rows, int cols, int count, std::string* why) {
    if (rows <= 0 || cols <= 0 || count <= 0) { *why = "rows, cols and count must be > 0"; return MUON_ERR_INVALID; }
    if ((long long)rows * cols > (1ll << 31) - 1) { *why = "a matrix may hold at most 2^31-1 elements"; return MUON_ERR_INVALID; }
    if (count > 65535) { *why = "count must be <= 65535"; return MUON_ERR_INVALID; }
    return MUON_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// A buffer of a call: [a, b) bytes, written or only read, and where it came from.
struct Span { uintptr_t a, b; bool written; int group, index; char what; };

// MUON_ERR_INVALID when a written span overlaps any other span (read-only spans may
// overlap each other).  One sort and one sweep: a span overlaps an earlier one
// exactly when it starts before the largest end seen so far.
muon_status check_spans(std::vector<Span>& sp, std::string* why) {
    std::sort(sp.begin(), sp.end(), [](const Span& x, const Span& y) { return x.a < y.a; });
    uintptr_t end_any = 0, end_written = 0;
    for (const Span& x : sp) {
        if (x.a < end_written || (x.written && x.a < end_any)) {
            *why = "group " + std::to_string(x.group) + ": " + x.what + "[" + std::to_string(x.index) +
                   "] overlaps a buffer that the call writes (written buffers may not share memory with any "
                   "other buffer of the call)";
            return MUON_ERR_INVALID;
        }
        end_any = std::max(end_any, x.b);
        if (x.written) end_written = std::max(end_written, x.b);
    }
    return MUON_OK;
}

muon_status check_groups(const muon_group* g, int n, std::string* why) {
    if (!g || n <= 0) { *why = "groups must be a non-empty array"; return MUON_ERR_INVALID; }
    long long total = 0;
    for (int i = 0; i < n; ++i) {
        muon_status s = check_shape(g[i].rows, g[i].cols, g[i].count, why);
        if (s != MUON_OK) { *why = "group " + std::to_string(i) + ": " + *why; return s; }
        if (g[i].grad_dtype != MUON_BF16 && g[i].grad_dtype != MUON_FP32) { *why = "group " + std::to_string(i) + ": bad grad_dtype"; return MUON_ERR_INVALID; }
        if (!finite(g[i].scale)) { *why = "group " + std::to_string(i) + ": scale is not finite"; return MUON_ERR_INVALID; }
        if (!g[i].W || !g[i].G || !g[i].B) { *why = "group " + std::to_string(i) + ": W, G and B arrays are required"; return MUON_ERR_INVALID; }
        for (int k = 0; k < g[i].count; ++k) {
            if (!g[i].W[k] || !g[i].G[k] || !g[i].B[k]) { *why = "group " + std::to_string(i) + ": NULL matrix pointer at index " + std::to_string(k); return MUON_ERR_INVALID; }
            if (!aligned(g[i].W[k], 4) || !aligned(g[i].B[k], 4) || !aligned(g[i].G[k], g[i].grad_dtype == MUON_BF16 ? 2 : 4)) {
                *why = "group " + std::to_string(i) + ": misaligned pointer at index " + std::to_string(k); return MUON_ERR_INVALID;
            }
        }
        total += g[i].count;
    }
    if (total > (1 << 24)) { *why = "too many matrices"; return MUON_ERR_INVALID; }
    // W and B are written in place: neither may overlap any other matrix's W, G or B
    // (G buffers are only read and may be shared).
    std::vector<Span> sp;
    sp.reserve((size_t)total * 3);
    for (int i = 0; i < n; ++i) {
        const uintptr_t e = (uintptr_t)g[i].rows * (uintptr_t)g[i].cols;
        const uintptr_t gb = e * (g[i].grad_dtype == MUON_BF16 ? 2 : 4);
        for (int k = 0; k < g[i].count; ++k) {
            const uintptr_t w = (uintptr_t)g[i].W[k], b = (uintptr_t)g[i].B[k], gg = (uintptr_t)g[i].G[k];
            sp.push_back(Span{w, w + 4 * e, true, i, k, 'W'});
            sp.push_back(Span{b, b + 4 * e, true, i, k, 'B'});
            sp.push_back(Span{gg, gg + gb, false, i, k, 'G'});
        }
    }
    return check_spans(sp, why);
}

muon_status ensure_buf(muon_handle* h, DevBuf& b, size_t bytes) {
    if (b.size >= bytes) return MUON_OK;
    if (b.ptr) {
        cudaError_t e = cudaDeviceSynchronize();   // the old buffer may still be in use
        if (e != cudaSuccess) return fail(h, MUON_ERR_CUDA, "cudaDeviceSynchronize: %s", cudaGetErrorString(e));
        cudaFree(b.ptr);
        b.ptr = nullptr;
        b.size = 0;
    }
    const size_t held = h->ws.size + h->staging.size + h->scratch.size + h->apply_segs.size;   // b is already released
    if (h->mem_limit != 0 && held + bytes > h->mem_limit)
        return fail(h, MUON_ERR_OOM, "device buffers of %zu bytes would exceed the handle's memory limit of %zu bytes",
                    held + bytes, h->mem_limit);
    cudaError_t e = cudaMalloc(&b.ptr, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        b.ptr = nullptr;
        return fail(h, MUON_ERR_OOM, "workspace allocation of %zu bytes failed: %s", bytes, cudaGetErrorString(e));
    }
    b.size = bytes;
    return MUON_OK;
}

muon_status load_encoder(muon_handle* h) {
    if (h->encode) return MUON_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
        return fail(h, MUON_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled is not available from the driver");
    h->encode = reinterpret_cast<EncodeTiledFn>(fn);
    return MUON_OK;
}

// 3-D bf16 tensor map over [count][rows][ld] with the logical width `cols`:
// box of box_cols (= 64, one 128-byte swizzle span) x box_rows, 128-byte swizzle,
// zero fill outside.
muon_status encode_map_box(muon_handle* h, CUtensorMap* m, const void* base, int cols, int rows, int count, int ld,
                           int box_cols, int box_rows, CUtensorMapSwizzle swz) {
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)count};
    cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)ld * 2 * (cuuint64_t)rows};
    cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = h->encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(h, MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for %dx%dx%d ld %d box %dx%d", (int)r, count,
                    rows, cols, ld, box_rows, box_cols);
    return MUON_OK;
}

muon_status encode_map(muon_handle* h, CUtensorMap* m, const void* base, int cols, int rows, int count, int ld,
                       int box_rows) {
    return encode_map_box(h, m, base, cols, rows, count, ld, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Boxes of the UPDATE epilogue: tc_gemm_epi_rows() x tc_gemm_epi_cols() (32 bf16
// columns, one 64-byte row), with the 64-byte swizzle whose span is one box row.
muon_status encode_epi_map(muon_handle* h, CUtensorMap* m, const void* base, int cols, int rows, int count, int ld) {
    return encode_map_box(h, m, base, cols, rows, count, ld, tc_gemm_epi_cols(), tc_gemm_epi_rows(),
                          tc_gemm_epi_cols() == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

// The two boxes of a symmetric m x m output (A or P) for the Gram / polynomial
// epilogue: [0] the direct box (as encode_epi_map), [1] its transpose, tc_gemm_epi_cols()
// rows of tc_gemm_epi_rows() columns, unswizzled, for the mirrored stores.
muon_status encode_sym_maps(muon_handle* h, CUtensorMap* m2, const void* base, int mdim, int count, int ld) {
    muon_status st = encode_epi_map(h, &m2[0], base, mdim, mdim, count, ld);
    if (st != MUON_OK) return st;
    return encode_map_box(h, &m2[1], base, mdim, mdim, count, ld, tc_gemm_epi_rows(), tc_gemm_epi_cols(),
                          CU_TENSOR_MAP_SWIZZLE_NONE);
}

bool is_bf16_path(const muon_handle* h) { return h->cfg.precision == MUON_PREC_BF16; }

// Persistent grid: one CTA (or one two-CTA cluster) per tile, at most one per SM.
// The two-CTA kernel runs one pair per unit list (lists are built for max_clusters).
// pair: two CTAs per cluster that has units (`active`, 0 = all clusters)
int gemm_grid(const muon_handle* h, int ntiles, int active = 0) {
    if (h->pair) return 2 * (active > 0 ? active : h->max_clusters);
    return std::min(ntiles, h->num_sms);
}

// Builds (or reuses) the plan for the shape list; allocates the workspace,
// writes tile lists, tensor maps and group descriptors to the device.
muon_status ensure_plan(muon_handle* h, const std::vector<int>& shapes, cudaStream_t s) {
    std::vector<int> key = shapes;
    key.push_back(h->cfg.precision);
    Plan& P = h->plan;
    if (P.valid && P.key == key) return MUON_OK;
    P = Plan();
    P.key = key;
    P.version = ++h->plans_built;
    const bool bf16 = is_bf16_path(h);
    const int ng = (int)shapes.size() / 3;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = align_up(off, 256); off = o + align_up(bytes, 256); return o; };
    int mat = 0, k1 = 0, k7 = 0;
    for (int g = 0; g < ng; ++g) {
        GroupDims d = make_dims(shapes[3 * g], shapes[3 * g + 1], shapes[3 * g + 2]);
        P.dims.push_back(d);
        P.mat_base.push_back(mat);
        GroupOffsets o{};
        const size_t xe = (size_t)d.count * d.m * d.ldn, ae = (size_t)d.count * d.m * d.ldm;
        if (bf16) {
            o.xb[0] = take(xe * 2); o.xb[1] = take(xe * 2);
            o.xl = take(xe * 2);
            o.xf[0] = o.xf[1] = 0;
            o.a = take(ae * 2); o.p = take(ae * 2);
        } else {
            o.xb[0] = o.xb[1] = o.xl = 0;
            o.xf[0] = take(xe * 4); o.xf[1] = take(xe * 4);
            o.a = take(ae * 4); o.p = take(ae * 4);
        }
        P.offs.push_back(o);
        for (int z = 0; z < d.count; ++z, ++mat) {
            EwSeg sg{};
            sg.rows = d.rows; sg.cols = d.cols; sg.ldn = d.ldn; sg.transposed = d.transposed;
            int nb, na;
            if (d.transposed) {
                nb = na = ((d.rows + MT_ROWS - 1) / MT_ROWS) * ((d.cols + MT_COLS - 1) / MT_COLS);
            } else {
                nb = na = (int)(((long long)d.rows * d.cols + EW_FLAT_ELEMS - 1) / EW_FLAT_ELEMS);
            }
            sg.blk_begin = k1; sg.blk_count = nb; k1 += nb;
            sg.apply_begin = k7; sg.apply_count = na; k7 += na;
            sg.mat = mat;
            P.segs.push_back(sg);
        }
    }
    P.nmat = mat;
    P.k1_blocks = k1;
    P.k7_blocks = k7;
    std::vector<Tile> tg, tp, tu;
    UnitPlan upl[3];
    int sk_slots = 0;
    if (bf16) {
        if (!h->tc_ready) {
            CUDA_TRY(h, tc_gemm_prepare());
            CUDA_TRY(h, tc_gemm_max_clusters(&h->max_clusters));
            if (h->max_clusters < 1) return fail(h, MUON_ERR_UNSUPPORTED, "no two-CTA cluster fits on this device");
            h->tc_ready = true;
        }
        const int bm = tc_gemm_tile_m(h->pair), bn = tc_gemm_tile_n(h->pair);
        tg = build_tiles(P.dims, 0, bm, bn);
        tp = build_tiles(P.dims, 1, bm, bn);
        tu = build_tiles(P.dims, 2, bm, bn);
        if (h->pair) {
            const std::vector<Tile>* lists[3] = {&tg, &tp, &tu};
            for (int ph = 0; ph < 3; ++ph) {
                std::vector<int> kb;
                for (const Tile& t : *lists[ph]) {
                    const GroupDims& d = P.dims[t.group];
                    kb.push_back(((ph == 0 ? d.n : d.m) + TC_BK - 1) / TC_BK);
                }
                upl[ph] = build_units(*lists[ph], kb, h->max_clusters, tc_gemm_split_tiles() != 0, true);
                sk_slots = std::max(sk_slots, upl[ph].nslots);
                P.active[ph] = active_clusters(upl[ph], h->max_clusters);
            }
            P.unit_clusters = h->max_clusters;
        }
        // per phase, the shared-memory configuration for the tiles' average K
        {
            const std::vector<Tile>* lists[3] = {&tg, &tp, &tu};
            const int modes[3] = {MODE_GRAM, MODE_POLY, MODE_UPDATE};
            for (int ph = 0; ph < 3; ++ph) {
                long long ksum = 0;
                for (const Tile& t : *lists[ph]) ksum += ph == 0 ? P.dims[t.group].n : P.dims[t.group].m;
                const int avg = lists[ph]->empty() ? 0 : (int)(ksum / (long long)lists[ph]->size());
                P.var[ph] = tc_gemm_var(modes[ph], avg);
            }
        }
        P.fused_apply = tc_gemm_fused_apply() != 0;
        // nothing is launched with a plan that does not cover its outputs exactly once
        const std::vector<Tile>* lists[3] = {&tg, &tp, &tu};
        for (int ph = 0; ph < 3; ++ph) {
            std::vector<int> kb;
            for (const Tile& t : *lists[ph]) {
                const GroupDims& d = P.dims[t.group];
                kb.push_back(((ph == 0 ? d.n : d.m) + TC_BK - 1) / TC_BK);
            }
            const std::string bad = check_plan(P.dims, ph, bm, bn, TC_BK, *lists[ph], kb,
                                               h->pair ? &upl[ph] : nullptr, h->pair ? h->max_clusters : 1);
            if (!bad.empty()) return fail(h, MUON_ERR_INVALID, "plan check failed (phase %d): %s", ph, bad.c_str());
        }
    }
    P.n_gram = (int)tg.size(); P.n_poly = (int)tp.size(); P.n_upd = (int)tu.size();
    const size_t o_tg = take(tg.size() * sizeof(int4) + 16), o_tp = take(tp.size() * sizeof(int4) + 16),
                 o_tu = take(tu.size() * sizeof(int4) + 16);
    const size_t o_maps = take(ng * sizeof(GemmMaps)), o_ginfo = take(ng * sizeof(GemmGroupInfo));
    const size_t o_segs = take(P.segs.size() * sizeof(EwSeg)), o_part = take((size_t)k1 * sizeof(double) + 8);
    const size_t o_norm = take((size_t)mat * sizeof(float)), o_scale = take((size_t)mat * sizeof(float));
    const size_t o_cnt = take((size_t)mat * sizeof(int));
    const size_t o_rmsp = take((size_t)mat * UPDATE_RMS_PARTIALS * sizeof(double)), o_rms = take((size_t)mat * sizeof(float));
    size_t o_units[3], o_ubeg[3];
    for (int ph = 0; ph < 3; ++ph) {
        o_units[ph] = take(upl[ph].units.size() * 2 * sizeof(int4) + 32);
        o_ubeg[ph] = take(upl[ph].begin.size() * sizeof(int) + 16);
    }
    const size_t o_skp = take((size_t)sk_slots * SK_SLOT_FLOATS * sizeof(float) + 16);
    const size_t o_skc = take((size_t)sk_slots * sizeof(int) + 16), o_skf = take((size_t)sk_slots * sizeof(int) + 16);
    muon_status st = ensure_buf(h, h->ws, off);
    if (st != MUON_OK) { P.valid = false; return st; }
    char* base = static_cast<char*>(h->ws.ptr);
    P.d_tiles_gram = reinterpret_cast<int4*>(base + o_tg);
    P.d_tiles_poly = reinterpret_cast<int4*>(base + o_tp);
    P.d_tiles_upd = reinterpret_cast<int4*>(base + o_tu);
    for (int ph = 0; ph < 3; ++ph) {
        P.d_units[ph] = reinterpret_cast<int4*>(base + o_units[ph]);
        P.d_unit_begin[ph] = reinterpret_cast<int*>(base + o_ubeg[ph]);
    }
    P.d_sk_partial = reinterpret_cast<float*>(base + o_skp);
    P.d_sk_count = reinterpret_cast<int*>(base + o_skc);
    P.d_sk_flag = reinterpret_cast<int*>(base + o_skf);
    if (sk_slots > 0) {
        CUDA_TRY(h, cudaMemsetAsync(P.d_sk_count, 0, (size_t)sk_slots * sizeof(int), s));
        CUDA_TRY(h, cudaMemsetAsync(P.d_sk_flag, 0, (size_t)sk_slots * sizeof(int), s));
    }
    P.d_maps = reinterpret_cast<GemmMaps*>(base + o_maps);
    P.d_ginfo = reinterpret_cast<GemmGroupInfo*>(base + o_ginfo);
    P.d_segs = reinterpret_cast<EwSeg*>(base + o_segs);
    P.d_partials = reinterpret_cast<double*>(base + o_part);
    P.d_norms = reinterpret_cast<float*>(base + o_norm);
    P.d_scale = reinterpret_cast<float*>(base + o_scale);
    P.d_counters = reinterpret_cast<int*>(base + o_cnt);
    P.d_rms_part = reinterpret_cast<double*>(base + o_rmsp);
    P.d_rms = reinterpret_cast<float*>(base + o_rms);
    CUDA_TRY(h, cudaMemsetAsync(P.d_counters, 0, (size_t)mat * sizeof(int), s));

    // workspace pointers in the segment table
    int mi = 0;
    for (int g = 0; g < ng; ++g) {
        const GroupDims& d = P.dims[g];
        const size_t xe = (size_t)d.m * d.ldn;
        for (int z = 0; z < d.count; ++z, ++mi) {
            EwSeg& sg = P.segs[mi];
            if (bf16) {
                sg.xhi0 = reinterpret_cast<__nv_bfloat16*>(base + P.offs[g].xb[0]) + (size_t)z * xe;
                sg.xlo0 = reinterpret_cast<__nv_bfloat16*>(base + P.offs[g].xl) + (size_t)z * xe;
            } else {
                sg.xf0 = reinterpret_cast<float*>(base + P.offs[g].xf[0]) + (size_t)z * xe;
            }
        }
    }
    if (bf16) {
        if ((st = load_encoder(h)) != MUON_OK) return st;
        std::vector<GemmMaps> maps(ng);
        std::vector<GemmGroupInfo> gi(ng);
        for (int g = 0; g < ng; ++g) {
            const GroupDims& d = P.dims[g];
            const GroupOffsets& o = P.offs[g];
            for (int b = 0; b < 2; ++b) {
                if ((st = encode_map(h, &maps[g].xb_k[b], base + o.xb[b], d.n, d.m, d.count, d.ldn, 128)) != MUON_OK) return st;
                if ((st = encode_map(h, &maps[g].xb_mn[b], base + o.xb[b], d.n, d.m, d.count, d.ldn, 64)) != MUON_OK) return st;
            }
            if ((st = encode_map(h, &maps[g].a, base + o.a, d.m, d.m, d.count, d.ldm, 128)) != MUON_OK) return st;
            if ((st = encode_map(h, &maps[g].p, base + o.p, d.m, d.m, d.count, d.ldm, 128)) != MUON_OK) return st;
            for (int b = 0; b < 2; ++b)
                if ((st = encode_epi_map(h, &maps[g].xe_hi[b], base + o.xb[b], d.n, d.m, d.count, d.ldn)) != MUON_OK) return st;
            if ((st = encode_epi_map(h, &maps[g].xe_lo_in, base + o.xl, d.n, d.m, d.count, d.ldn)) != MUON_OK) return st;
            maps[g].xe_lo_out = maps[g].xe_lo_in;
            if ((st = encode_sym_maps(h, maps[g].se_a, base + o.a, d.m, d.count, d.ldm)) != MUON_OK) return st;
            if ((st = encode_sym_maps(h, maps[g].se_p, base + o.p, d.m, d.count, d.ldm)) != MUON_OK) return st;
            GemmGroupInfo& q = gi[g];
            q.m = d.m; q.n = d.n; q.ldm = d.ldm; q.ldn = d.ldn; q.count = d.count; q.mat_base = P.mat_base[g];
            q.xb[0] = reinterpret_cast<__nv_bfloat16*>(base + o.xb[0]);
            q.xb[1] = reinterpret_cast<__nv_bfloat16*>(base + o.xb[1]);
            q.xlo_in = reinterpret_cast<const __nv_bfloat16*>(base + o.xl);
            q.xlo_out = reinterpret_cast<__nv_bfloat16*>(base + o.xl);
            q.a = reinterpret_cast<__nv_bfloat16*>(base + o.a);
            q.p = reinterpret_cast<__nv_bfloat16*>(base + o.p);
        }
        auto up_tiles = [&](int4* dst, const std::vector<Tile>& t) -> cudaError_t {
            if (t.empty()) return cudaSuccess;
            std::vector<int4> v(t.size());
            for (size_t i = 0; i < t.size(); ++i) v[i] = make_int4(t[i].group, t[i].mat, t[i].tile_row, t[i].tile_col);
            return cudaMemcpyAsync(dst, v.data(), v.size() * sizeof(int4), cudaMemcpyHostToDevice, s);
        };
        CUDA_TRY(h, up_tiles(P.d_tiles_gram, tg));
        CUDA_TRY(h, up_tiles(P.d_tiles_poly, tp));
        CUDA_TRY(h, up_tiles(P.d_tiles_upd, tu));
        std::vector<std::vector<int4>> uv(3);
        for (int ph = 0; ph < 3 && h->pair; ++ph) {
            for (const Unit& u : upl[ph].units) {
                uv[ph].push_back(make_int4(u.tile.group, u.tile.mat, u.tile.tile_row, u.tile.tile_col));
                uv[ph].push_back(make_int4(u.k_begin, u.k_end, u.kind | (u.n_half << 8), u.slot | (u.nslots << 16)));
            }
            if (!uv[ph].empty())
                CUDA_TRY(h, cudaMemcpyAsync(P.d_units[ph], uv[ph].data(), uv[ph].size() * sizeof(int4),
                                            cudaMemcpyHostToDevice, s));
            CUDA_TRY(h, cudaMemcpyAsync(P.d_unit_begin[ph], upl[ph].begin.data(), upl[ph].begin.size() * sizeof(int),
                                        cudaMemcpyHostToDevice, s));
        }
        CUDA_TRY(h, cudaMemcpyAsync(P.d_maps, maps.data(), ng * sizeof(GemmMaps), cudaMemcpyHostToDevice, s));
        CUDA_TRY(h, cudaMemcpyAsync(P.d_ginfo, gi.data(), ng * sizeof(GemmGroupInfo), cudaMemcpyHostToDevice, s));
        // pageable copies are staged before return; wait so the host vectors may go
        CUDA_TRY(h, cudaStreamSynchronize(s));
    }
    P.valid = true;
    return MUON_OK;
}

float update_scale(const muon_handle* h, int rows, int cols, float custom) {
    switch (h->cfg.scale_mode) {
        case MUON_SCALE_MATCH_RMS: return h->cfg.rms_target * std::sqrt((float)(rows > cols ? rows : cols));
        case MUON_SCALE_CUSTOM: return custom;
        default: return 1.0f;
    }
}

// Fills the caller-pointer part of the segment table and uploads it if it changed.
struct MatPtrs { const void* g; float* b; float* w; int g_bf16; float scale; int out_bf16 = 0; };

muon_status upload_segs(muon_handle* h, const std::vector<MatPtrs>& mp, cudaStream_t s) {
    Plan& P = h->plan;
    const bool bf16 = is_bf16_path(h);
    std::vector<EwSeg> segs = P.segs;
    int mi = 0;
    char* base = static_cast<char*>(h->ws.ptr);
    for (size_t g = 0; g < P.dims.size(); ++g) {
        const GroupDims& d = P.dims[g];
        const size_t xe = (size_t)d.m * d.ldn;
        const int final_buf = bf16 ? 0 : (h->cfg.ns_steps & 1);
        for (int z = 0; z < d.count; ++z, ++mi) {
            EwSeg& sg = segs[mi];
            sg.g = mp[mi].g; sg.b = mp[mi].b; sg.w = mp[mi].w;
            sg.g_bf16 = mp[mi].g_bf16;
            sg.update_scale = mp[mi].scale;
            sg.out_bf16 = mp[mi].out_bf16;
            if (bf16) {
                sg.o_hi = reinterpret_cast<const __nv_bfloat16*>(base + P.offs[g].xb[h->cfg.ns_steps & 1]) + (size_t)z * xe;
                sg.o_lo = reinterpret_cast<const __nv_bfloat16*>(base + P.offs[g].xl) + (size_t)z * xe;
            } else {
                sg.o_src = reinterpret_cast<const float*>(base + P.offs[g].xf[final_buf]) + (size_t)z * xe;
            }
            sg.vec = (d.cols % 8 == 0) && aligned(sg.g, 16) && aligned(sg.w, 16) && (sg.b == nullptr || aligned(sg.b, 16)) ? 1 : 0;
        }
    }
    if (P.uploaded.size() == segs.size() && std::memcmp(P.uploaded.data(), segs.data(), segs.size() * sizeof(EwSeg)) == 0)
        return MUON_OK;
    CUDA_TRY(h, cudaMemcpyAsync(P.d_segs, segs.data(), segs.size() * sizeof(EwSeg), cudaMemcpyHostToDevice, s));
    CUDA_TRY(h, cudaStreamSynchronize(s));
    P.uploaded = segs;
    return MUON_OK;
}

// Work that muon_step_host splices into the launch sequence.
struct Hooks {
    cudaEvent_t w_ready = nullptr;                    // s waits for it before W is first read
    std::function<muon_status()> after_momentum;     // enqueued right after the momentum kernel
};

muon_status run_pipeline(muon_handle* h, bool momentum, bool copy_out, cudaStream_t s, const Hooks* hooks = nullptr) {
    Plan& P = h->plan;
    const muon_config& c = h->cfg;
    const bool bf16 = is_bf16_path(h);
    TIMED(h, 0, s, launch_momentum_norm(P.d_segs, P.nmat, P.k1_blocks, P.d_partials, momentum ? c.momentum : 0.f,
                                        momentum ? c.nesterov : 0, bf16 ? 1 : 0, P.d_counters, c.eps, P.d_norms,
                                        P.d_scale, s));
    if (hooks && hooks->after_momentum) {
        muon_status st = hooks->after_momentum();
        if (st != MUON_OK) return st;
    }
    char* base = static_cast<char*>(h->ws.ptr);
    for (int it = 0; it < c.ns_steps; ++it) {
        const int par = it & 1;
        if (bf16) {
            GemmParams gp{};
            gp.maps = P.d_maps; gp.groups = P.d_ginfo; gp.parity = par; gp.err = h->d_err;
            gp.sk_partial = P.d_sk_partial; gp.sk_count = P.d_sk_count; gp.sk_flag = P.d_sk_flag;
            gp.tiles = P.d_tiles_gram; gp.ntiles = P.n_gram; gp.alpha = 1.f; gp.beta = 0.f;
            gp.units = P.d_units[0]; gp.unit_begin = P.d_unit_begin[0]; gp.epoch = ++h->epoch;
            gp.scale = it == 0 ? P.d_scale : nullptr;
            TIMED(h, 2, s, launch_tc_gemm(MODE_GRAM, h->pair, gp, gemm_grid(h, P.n_gram, P.active[0]), s, P.var[0]));
            gp.tiles = P.d_tiles_poly; gp.ntiles = P.n_poly; gp.alpha = c.ns_c; gp.beta = c.ns_b; gp.scale = nullptr;
            gp.units = P.d_units[1]; gp.unit_begin = P.d_unit_begin[1]; gp.epoch = ++h->epoch;
            TIMED(h, 3, s, launch_tc_gemm(MODE_POLY, h->pair, gp, gemm_grid(h, P.n_poly, P.active[1]), s, P.var[1]));
            gp.tiles = P.d_tiles_upd; gp.ntiles = P.n_upd; gp.alpha = 1.f; gp.beta = c.ns_a;
            gp.units = P.d_units[2]; gp.unit_begin = P.d_unit_begin[2]; gp.epoch = ++h->epoch;
            gp.scale = it == 0 ? P.d_scale : nullptr;
            if (it + 1 == c.ns_steps && P.fused_apply) {        // fused apply / copy-out
                if (hooks && hooks->w_ready) CUDA_TRY(h, cudaStreamWaitEvent(s, hooks->w_ready, 0));
                gp.apply_mode = copy_out ? 2 : 1;
                gp.decay = copy_out ? 1.f : 1.f - c.lr * c.weight_decay;
                gp.lr = c.lr;
                gp.segs = P.d_segs;
            }
            TIMED(h, 4, s, launch_tc_gemm(MODE_UPDATE, h->pair, gp, gemm_grid(h, P.n_upd, P.active[2]), s, P.var[2]));
        } else {
            for (size_t g = 0; g < P.dims.size(); ++g) {
                const GroupDims& d = P.dims[g];
                const GroupOffsets& o = P.offs[g];
                float* x_cur = reinterpret_cast<float*>(base + o.xf[par]);
                float* x_nxt = reinterpret_cast<float*>(base + o.xf[par ^ 1]);
                float* A = reinterpret_cast<float*>(base + o.a);
                float* Pm = reinterpret_cast<float*>(base + o.p);
                const long long sx = (long long)d.m * d.ldn, sa = (long long)d.m * d.ldm;
                SimtGemmArgs ga{};
                ga.A = x_cur; ga.B = x_cur; ga.C = A; ga.Cin = nullptr;
                ga.M = d.m; ga.N = d.m; ga.K = d.n; ga.lda = d.ldn; ga.ldb = d.ldn; ga.ldc = d.ldm; ga.ldcin = 0;
                ga.sA = sx; ga.sB = sx; ga.sC = sa; ga.sCin = 0; ga.count = d.count; ga.b_kmajor = 1;
                ga.alpha = 1.f; ga.beta = 0.f; ga.scale = it == 0 ? P.d_scale : nullptr; ga.scale_pow = 2;
                ga.mat_base = P.mat_base[g];
                TIMED(h, 2, s, launch_simt_gemm(ga, s));
                SimtGemmArgs gb{};
                gb.A = A; gb.B = A; gb.C = Pm; gb.Cin = A;
                gb.M = d.m; gb.N = d.m; gb.K = d.m; gb.lda = d.ldm; gb.ldb = d.ldm; gb.ldc = d.ldm; gb.ldcin = d.ldm;
                gb.sA = sa; gb.sB = sa; gb.sC = sa; gb.sCin = sa; gb.count = d.count; gb.b_kmajor = 1;
                gb.alpha = c.ns_c; gb.beta = c.ns_b; gb.scale = nullptr; gb.scale_pow = 0; gb.mat_base = P.mat_base[g];
                TIMED(h, 3, s, launch_simt_gemm(gb, s));
                SimtGemmArgs gu{};
                gu.A = Pm; gu.B = x_cur; gu.C = x_nxt; gu.Cin = x_cur;
                gu.M = d.m; gu.N = d.n; gu.K = d.m; gu.lda = d.ldm; gu.ldb = d.ldn; gu.ldc = d.ldn; gu.ldcin = d.ldn;
                gu.sA = sa; gu.sB = sx; gu.sC = sx; gu.sCin = sx; gu.count = d.count; gu.b_kmajor = 0;
                gu.alpha = 1.f; gu.beta = c.ns_a; gu.scale = it == 0 ? P.d_scale : nullptr; gu.scale_pow = 1;
                gu.mat_base = P.mat_base[g];
                TIMED(h, 4, s, launch_simt_gemm(gu, s));
            }
        }
    }
    if (bf16 && c.ns_steps > 0 && P.fused_apply) return MUON_OK;
    if (hooks && hooks->w_ready) CUDA_TRY(h, cudaStreamWaitEvent(s, hooks->w_ready, 0));
    const float decay = copy_out ? 1.f : 1.f - c.lr * c.weight_decay;
    TIMED(h, 5, s, launch_apply(P.d_segs, P.nmat, P.k7_blocks, decay, c.lr, c.ns_steps == 0 ? P.d_scale : nullptr,
                                copy_out ? 1 : 0, s));
    return MUON_OK;
}

// Replays the captured launch sequence when nothing it depends on has changed,
// else captures it again on a private stream (graph capture is not allowed on the
// legacy default stream).  Direct launches when timing is on, when the host-buffer
// step splices copies in, when the caller's stream is itself being captured, or when
// split tiles are used (their flags carry a per-launch epoch).
muon_status run_graph_or_direct(muon_handle* h, bool momentum, bool copy_out, cudaStream_t s, const Hooks* hooks) {
    Plan& P = h->plan;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    CUDA_TRY(h, cudaStreamIsCapturing(s, &cs));
    const bool use_graph = h->graphs && !h->timing && !hooks && cs == cudaStreamCaptureStatusNone &&
                           !(h->pair && tc_gemm_split_tiles());
    if (!use_graph) return run_pipeline(h, momentum, copy_out, s, hooks);
    const int mode = (copy_out ? 1 : 0) | (momentum ? 2 : 0);
    const bool same = h->gexec && h->g_mode == mode && h->g_ws == h->ws.ptr && h->g_version == P.version &&
                      std::memcmp(&h->g_cfg, &h->cfg, sizeof(muon_config)) == 0 && h->g_segs.size() == P.uploaded.size() &&
                      std::memcmp(h->g_segs.data(), P.uploaded.data(), P.uploaded.size() * sizeof(EwSeg)) == 0;
    if (!same) {
        if (h->gexec) { cudaGraphExecDestroy(h->gexec); h->gexec = nullptr; }
        if (!h->cap_stream) CUDA_TRY(h, cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking));
        CUDA_TRY(h, cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal));
        muon_status st = run_pipeline(h, momentum, copy_out, h->cap_stream, nullptr);
        cudaGraph_t graph = nullptr;
        cudaError_t e = cudaStreamEndCapture(h->cap_stream, &graph);
        if (st != MUON_OK) { if (graph) cudaGraphDestroy(graph); return st; }
        if (e != cudaSuccess) return fail(h, MUON_ERR_CUDA, "graph capture failed: %s", cudaGetErrorString(e));
        e = cudaGraphInstantiate(&h->gexec, graph, 0);
        cudaGraphDestroy(graph);
        if (e != cudaSuccess) { h->gexec = nullptr; return fail(h, MUON_ERR_CUDA, "graph instantiation failed: %s", cudaGetErrorString(e)); }
        h->g_mode = mode;
        h->g_ws = h->ws.ptr;
        h->g_version = P.version;
        h->g_cfg = h->cfg;
        h->g_segs = P.uploaded;
    }
    CUDA_TRY(h, cudaGraphLaunch(h->gexec, s));
    return MUON_OK;
}

muon_status step_device(muon_handle* h, const muon_group* groups, int n, cudaStream_t s,
                        const Hooks* hooks = nullptr) {
    std::vector<int> shapes;
    std::vector<MatPtrs> mp;
    for (int i = 0; i < n; ++i) {
        shapes.push_back(groups[i].rows); shapes.push_back(groups[i].cols); shapes.push_back(groups[i].count);
        const float sc = update_scale(h, groups[i].rows, groups[i].cols, groups[i].scale);
        for (int k = 0; k < groups[i].count; ++k)
            mp.push_back(MatPtrs{groups[i].G[k], groups[i].B[k], groups[i].W[k], groups[i].grad_dtype == MUON_BF16 ? 1 : 0, sc});
    }
    muon_status st = ensure_plan(h, shapes, s);
    if (st != MUON_OK) return st;
    if ((st = upload_segs(h, mp, s)) != MUON_OK) return st;
    return run_graph_or_direct(h, true, false, s, hooks);
}

}  // namespace

// ============================================================================ C ABI

extern "C" {

void muon_config_default(muon_config* c) {
    if (!c) return;
    std::memset(c, 0, sizeof(*c));
    c->lr = 0.02f;
    c->momentum = 0.95f;
    c->weight_decay = 0.f;
    c->eps = 1e-7f;
    c->rms_target = 0.2f;
    c->nesterov = 1;
    c->ns_steps = 5;
    c->ns_a = 3.4445f;
    c->ns_b = -4.7750f;
    c->ns_c = 2.0315f;
    c->scale_mode = MUON_SCALE_NONE;
    c->precision = MUON_PREC_BF16;
}

muon_status muon_validate_config(const muon_config* cfg) {
    std::string why;
    return check_config(cfg, &why);
}

muon_status muon_validate_groups(const muon_group* groups, int n_groups) {
    std::string why;
    return check_groups(groups, n_groups, &why);
}

muon_status muon_create(const muon_config* cfg, int device, muon_handle** out) {
    if (!out) return MUON_ERR_INVALID;
    std::string why;
    if (check_config(cfg, &why) != MUON_OK) return MUON_ERR_INVALID;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess) { cudaGetLastError(); return MUON_ERR_CUDA; }
    if (device < 0 || device >= ndev) return MUON_ERR_INVALID;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return MUON_ERR_CUDA;
    if (prop.major != 10 || prop.minor != 0) return MUON_ERR_UNSUPPORTED;   // built for sm_100a only
    muon_handle* h = new muon_handle();
    h->cfg = *cfg;
    h->device = device;
    h->num_sms = prop.multiProcessorCount;
    h->pair = tc_gemm_default_pair();
    {
        const char* v = std::getenv("MUON_GRAPHS");
        h->graphs = !(v && std::strcmp(v, "0") == 0);
    }
    DeviceGuard dg(device);
    if (cudaMalloc(&h->d_err, sizeof(int)) != cudaSuccess || cudaMemset(h->d_err, 0, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        delete h;
        return MUON_ERR_OOM;
    }
    *out = h;
    return MUON_OK;
}

muon_status muon_set_config(muon_handle* h, const muon_config* cfg) {
    if (!h) return MUON_ERR_INVALID;
    std::string why;
    if (check_config(cfg, &why) != MUON_OK) return fail(h, MUON_ERR_INVALID, "%s", why.c_str());
    const bool plan_changes = cfg->precision != h->cfg.precision;
    h->cfg = *cfg;
    if (plan_changes) h->plan.valid = false;
    h->plan.uploaded.clear();     // ns_steps / scale may change the segment table
    return MUON_OK;
}

muon_status muon_set_memory_limit(muon_handle* h, size_t bytes) {
    if (!h) return MUON_ERR_INVALID;
    h->mem_limit = bytes;
    return MUON_OK;
}

muon_status muon_memory_held(const muon_handle* h, size_t* bytes) {
    if (!h || !bytes) return MUON_ERR_INVALID;
    *bytes = h->ws.size + h->staging.size + h->scratch.size + h->apply_segs.size;
    return MUON_OK;
}

muon_status muon_step(muon_handle* h, const muon_group* groups, int n_groups, void* stream) {
    if (!h) return MUON_ERR_INVALID;
    NvtxRange nr("muon_step");
    std::string why;
    if (check_groups(groups, n_groups, &why) != MUON_OK) return fail(h, MUON_ERR_INVALID, "%s", why.c_str());
    DeviceGuard dg(h->device);
    h->last_error.clear();
    return step_device(h, groups, n_groups, static_cast<cudaStream_t>(stream));
}

muon_status muon_step_host(muon_handle* h, const muon_group* groups, int n_groups, void* stream) {
    if (!h) return MUON_ERR_INVALID;
    NvtxRange nr("muon_step_host");
    std::string why;
    if (check_groups(groups, n_groups, &why) != MUON_OK) return fail(h, MUON_ERR_INVALID, "%s", why.c_str());
    DeviceGuard dg(h->device);
    h->last_error.clear();
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // staging layout: per matrix W, B (fp32) and G
    size_t off = 0;
    std::vector<size_t> ow, ob, og;
    for (int i = 0; i < n_groups; ++i) {
        const size_t e = (size_t)groups[i].rows * groups[i].cols;
        const size_t gsz = e * (groups[i].grad_dtype == MUON_BF16 ? 2 : 4);
        for (int k = 0; k < groups[i].count; ++k) {
            ow.push_back(off); off = align_up(off + e * 4, 256);
            ob.push_back(off); off = align_up(off + e * 4, 256);
            og.push_back(off); off = align_up(off + gsz, 256);
        }
    }
    muon_status st = ensure_buf(h, h->staging, off);
    if (st != MUON_OK) return st;
    char* base = static_cast<char*>(h->staging.ptr);
    std::vector<std::vector<float*>> Wd(n_groups), Bd(n_groups);
    std::vector<std::vector<const void*>> Gd(n_groups);
    std::vector<muon_group> dg_groups(groups, groups + n_groups);
    if (!h->side) {
        CUDA_TRY(h, cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking));
        CUDA_TRY(h, cudaStreamCreateWithFlags(&h->side2, cudaStreamNonBlocking));
        cudaEvent_t* evs[4] = {&h->ev_start, &h->ev_w, &h->ev_k1, &h->ev_done};
        for (cudaEvent_t* e : evs) CUDA_TRY(h, cudaEventCreateWithFlags(e, cudaEventDisableTiming));
    }
    // G and B go up first, on s, with the whole host-to-device bandwidth: the momentum
    // kernel needs them.  W goes up afterwards on one side stream, while the
    // Newton-Schulz GEMMs run, and is waited for only before the weight update; B comes
    // back on a second side stream as soon as the momentum kernel has finished with it,
    // in the other direction of the link, so that it overlaps W's upload.  Both side
    // streams start after everything already queued on s (the staging area may still be
    // in use by the previous call).
    int mi = 0;
    for (int i = 0; i < n_groups; ++i) {
        const size_t e = (size_t)groups[i].rows * groups[i].cols;
        const size_t gsz = e * (groups[i].grad_dtype == MUON_BF16 ? 2 : 4);
        for (int k = 0; k < groups[i].count; ++k, ++mi) {
            float* w = reinterpret_cast<float*>(base + ow[mi]);
            float* b = reinterpret_cast<float*>(base + ob[mi]);
            void* g = base + og[mi];
            CUDA_TRY(h, cudaMemcpyAsync(g, groups[i].G[k], gsz, cudaMemcpyHostToDevice, s));
            CUDA_TRY(h, cudaMemcpyAsync(b, groups[i].B[k], e * 4, cudaMemcpyHostToDevice, s));
            Wd[i].push_back(w); Bd[i].push_back(b); Gd[i].push_back(g);
        }
        dg_groups[i].W = Wd[i].data(); dg_groups[i].B = Bd[i].data(); dg_groups[i].G = Gd[i].data();
    }
    CUDA_TRY(h, cudaEventRecord(h->ev_start, s));
    CUDA_TRY(h, cudaStreamWaitEvent(h->side, h->ev_start, 0));
    mi = 0;
    for (int i = 0; i < n_groups; ++i) {
        const size_t e = (size_t)groups[i].rows * groups[i].cols;
        for (int k = 0; k < groups[i].count; ++k, ++mi)
            CUDA_TRY(h, cudaMemcpyAsync(base + ow[mi], groups[i].W[k], e * 4, cudaMemcpyHostToDevice, h->side));
    }
    CUDA_TRY(h, cudaEventRecord(h->ev_w, h->side));
    Hooks hooks;
    hooks.w_ready = h->ev_w;
    hooks.after_momentum = [&]() -> muon_status {
        CUDA_TRY(h, cudaEventRecord(h->ev_k1, s));
        CUDA_TRY(h, cudaStreamWaitEvent(h->side2, h->ev_k1, 0));
        int j = 0;
        for (int i = 0; i < n_groups; ++i) {
            const size_t e = (size_t)groups[i].rows * groups[i].cols;
            for (int k = 0; k < groups[i].count; ++k, ++j)
                CUDA_TRY(h, cudaMemcpyAsync(groups[i].B[k], base + ob[j], e * 4, cudaMemcpyDeviceToHost, h->side2));
        }
        CUDA_TRY(h, cudaEventRecord(h->ev_done, h->side2));
        return MUON_OK;
    };
    if ((st = step_device(h, dg_groups.data(), n_groups, s, &hooks)) != MUON_OK) return st;
    mi = 0;
    for (int i = 0; i < n_groups; ++i) {
        const size_t e = (size_t)groups[i].rows * groups[i].cols;
        for (int k = 0; k < groups[i].count; ++k, ++mi)
            CUDA_TRY(h, cudaMemcpyAsync(groups[i].W[k], base + ow[mi], e * 4, cudaMemcpyDeviceToHost, s));
    }
    CUDA_TRY(h, cudaStreamWaitEvent(s, h->ev_done, 0));
    return MUON_OK;
}

muon_status muon_step_direction(muon_handle* h, const muon_direction_group* groups, int n_groups, void* stream) {
    if (!h) return MUON_ERR_INVALID;
    NvtxRange nr("muon_step_direction");
    if (!groups || n_groups <= 0) return fail(h, MUON_ERR_INVALID, "groups must be a non-empty array");
    std::vector<int> shapes;
    std::vector<MatPtrs> mp;
    std::vector<Span> sp;
    long long total = 0;
    for (int i = 0; i < n_groups; ++i) {
        const muon_direction_group& g = groups[i];
        std::string why;
        if (check_shape(g.rows, g.cols, g.count, &why) != MUON_OK) return fail(h, MUON_ERR_INVALID, "group %d: %s", i, why.c_str());
        if (g.grad_dtype != MUON_BF16 && g.grad_dtype != MUON_FP32) return fail(h, MUON_ERR_INVALID, "group %d: bad grad_dtype", i);
        if (g.out_dtype != MUON_BF16 && g.out_dtype != MUON_FP32) return fail(h, MUON_ERR_INVALID, "group %d: bad out_dtype", i);
        if (!g.G || !g.B || !g.O) return fail(h, MUON_ERR_INVALID, "group %d: G, B and O arrays are required", i);
        total += g.count;
        if (total > (1 << 24)) return fail(h, MUON_ERR_INVALID, "too many matrices");
        shapes.push_back(g.rows); shapes.push_back(g.cols); shapes.push_back(g.count);
        const uintptr_t e = (uintptr_t)g.rows * (uintptr_t)g.cols;
        const size_t gsz = g.grad_dtype == MUON_BF16 ? 2 : 4, osz = g.out_dtype == MUON_BF16 ? 2 : 4;
        for (int k = 0; k < g.count; ++k) {
            if (!g.G[k] || !g.B[k] || !g.O[k]) return fail(h, MUON_ERR_INVALID, "group %d: NULL pointer at %d", i, k);
            if (!aligned(g.B[k], 4) || !aligned(g.G[k], gsz) || !aligned(g.O[k], osz))
                return fail(h, MUON_ERR_INVALID, "group %d: misaligned pointer at %d", i, k);
            const uintptr_t b = (uintptr_t)g.B[k], gg = (uintptr_t)g.G[k], o = (uintptr_t)g.O[k];
            sp.push_back(Span{b, b + 4 * e, true, i, k, 'B'});
            sp.push_back(Span{o, o + osz * e, true, i, k, 'O'});
            sp.push_back(Span{gg, gg + gsz * e, false, i, k, 'G'});
            MatPtrs m{g.G[k], g.B[k], reinterpret_cast<float*>(g.O[k]), g.grad_dtype == MUON_BF16 ? 1 : 0, 1.0f,
                      g.out_dtype == MUON_BF16 ? 1 : 0};
            mp.push_back(m);
        }
    }
    {
        std::string why;
        if (check_spans(sp, &why) != MUON_OK) return fail(h, MUON_ERR_INVALID, "%s", why.c_str());
    }
    DeviceGuard dg(h->device);
    h->last_error.clear();
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    muon_status st = ensure_plan(h, shapes, s);
    if (st != MUON_OK) return st;
    if ((st = upload_segs(h, mp, s)) != MUON_OK) return st;
    return run_graph_or_direct(h, true, true, s, nullptr);
}

muon_status muon_apply(muon_handle* h, const muon_apply_group* groups, int n_groups, void* stream) {
    if (!h) return MUON_ERR_INVALID;
    NvtxRange nr("muon_apply");
    if (!groups || n_groups <= 0) return fail(h, MUON_ERR_INVALID, "groups must be a non-empty array");
    std::vector<EwSeg> segs;
    std::vector<Span> sp;
    int blocks = 0;
    for (int i = 0; i < n_groups; ++i) {
        const muon_apply_group& g = groups[i];
        std::string why;
        if (check_shape(g.rows, g.cols, g.count, &why) != MUON_OK) return fail(h, MUON_ERR_INVALID, "group %d: %s", i, why.c_str());
        if (g.o_dtype != MUON_BF16 && g.o_dtype != MUON_FP32) return fail(h, MUON_ERR_INVALID, "group %d: bad o_dtype", i);
        if (!finite(g.scale)) return fail(h, MUON_ERR_INVALID, "group %d: scale is not finite", i);
        if (!g.W || !g.O) return fail(h, MUON_ERR_INVALID, "group %d: W and O arrays are required", i);
        const uintptr_t e = (uintptr_t)g.rows * (uintptr_t)g.cols;
        const size_t osz = g.o_dtype == MUON_BF16 ? 2 : 4;
        const float sc = update_scale(h, g.rows, g.cols, g.scale);
        const int nb = (int)((e + EW_FLAT_ELEMS - 1) / EW_FLAT_ELEMS);
        for (int k = 0; k < g.count; ++k) {
            if (!g.W[k] || !g.O[k]) return fail(h, MUON_ERR_INVALID, "group %d: NULL pointer at %d", i, k);
            if (!aligned(g.W[k], 4) || !aligned(g.O[k], osz)) return fail(h, MUON_ERR_INVALID, "group %d: misaligned pointer at %d", i, k);
            if ((long long)blocks + nb > (1ll << 31) - 1) return fail(h, MUON_ERR_INVALID, "too many elements");
            const uintptr_t w = (uintptr_t)g.W[k], o = (uintptr_t)g.O[k];
            sp.push_back(Span{w, w + 4 * e, true, i, k, 'W'});
            sp.push_back(Span{o, o + osz * e, false, i, k, 'O'});
            EwSeg sg{};
            sg.w = g.W[k];
            if (g.o_dtype == MUON_BF16) sg.o_hi = static_cast<const __nv_bfloat16*>(g.O[k]);
            else sg.o_src = static_cast<const float*>(g.O[k]);
            sg.rows = g.rows; sg.cols = g.cols; sg.ldn = g.cols; sg.transposed = 0;
            sg.vec = (g.cols % 8 == 0) && aligned(g.W[k], 16) && aligned(g.O[k], 16) ? 1 : 0;
            sg.apply_begin = blocks; sg.apply_count = nb; blocks += nb;
            sg.mat = (int)segs.size();
            sg.update_scale = sc;
            segs.push_back(sg);
        }
    }
    {
        std::string why;
        if (check_spans(sp, &why) != MUON_OK) return fail(h, MUON_ERR_INVALID, "%s", why.c_str());
    }
    DeviceGuard dg(h->device);
    h->last_error.clear();
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool same = h->apply_uploaded.size() == segs.size() &&
                      std::memcmp(h->apply_uploaded.data(), segs.data(), segs.size() * sizeof(EwSeg)) == 0;
    if (!same) {
        // the table may still be read by an earlier launch on another stream
        if (h->apply_segs.ptr) CUDA_TRY(h, cudaDeviceSynchronize());
        muon_status st = ensure_buf(h, h->apply_segs, segs.size() * sizeof(EwSeg));
        if (st != MUON_OK) return st;
        CUDA_TRY(h, cudaMemcpyAsync(h->apply_segs.ptr, segs.data(), segs.size() * sizeof(EwSeg), cudaMemcpyHostToDevice, s));
        CUDA_TRY(h, cudaStreamSynchronize(s));
        h->apply_uploaded = segs;
    }
    const muon_config& c = h->cfg;
    TIMED(h, 5, s, launch_apply(static_cast<const EwSeg*>(h->apply_segs.ptr), (int)segs.size(), blocks,
                                1.f - c.lr * c.weight_decay, c.lr, nullptr, 0, s));
    return MUON_OK;
}

muon_status muon_orthogonalize(muon_handle* h, const muon_ortho_group* groups, int n_groups, void* stream) {
    if (!h) return MUON_ERR_INVALID;
    NvtxRange nr("muon_orthogonalize");
    if (!groups || n_groups <= 0) return fail(h, MUON_ERR_INVALID, "groups must be a non-empty array");
    std::vector<int> shapes;
    std::vector<MatPtrs> mp;
    for (int i = 0; i < n_groups; ++i) {
        std::string why;
        if (check_shape(groups[i].rows, groups[i].cols, groups[i].count, &why) != MUON_OK)
            return fail(h, MUON_ERR_INVALID, "group %d: %s", i, why.c_str());
        if (groups[i].in_dtype != MUON_BF16 && groups[i].in_dtype != MUON_FP32) return fail(h, MUON_ERR_INVALID, "group %d: bad in_dtype", i);
        if (!groups[i].M || !groups[i].O) return fail(h, MUON_ERR_INVALID, "group %d: M and O arrays are required", i);
        shapes.push_back(groups[i].rows); shapes.push_back(groups[i].cols); shapes.push_back(groups[i].count);
        for (int k = 0; k < groups[i].count; ++k) {
            if (!groups[i].M[k] || !groups[i].O[k]) return fail(h, MUON_ERR_INVALID, "group %d: NULL pointer at %d", i, k);
            if (!aligned(groups[i].O[k], 4) || !aligned(groups[i].M[k], groups[i].in_dtype == MUON_BF16 ? 2 : 4))
                return fail(h, MUON_ERR_INVALID, "group %d: misaligned pointer at %d", i, k);
            mp.push_back(MatPtrs{groups[i].M[k], nullptr, groups[i].O[k], groups[i].in_dtype == MUON_BF16 ? 1 : 0, 1.0f});
        }
    }
    {
        // O is written: it may not overlap any M or O of the call
        std::vector<Span> sp;
        for (int i = 0; i < n_groups; ++i) {
            const uintptr_t e = (uintptr_t)groups[i].rows * (uintptr_t)groups[i].cols;
            const uintptr_t mb = e * (groups[i].in_dtype == MUON_BF16 ? 2 : 4);
            for (int k = 0; k < groups[i].count; ++k) {
                const uintptr_t m = (uintptr_t)groups[i].M[k], o = (uintptr_t)groups[i].O[k];
                sp.push_back(Span{m, m + mb, false, i, k, 'M'});
                sp.push_back(Span{o, o + 4 * e, true, i, k, 'O'});
            }
        }
        std::string why;
        if (check_spans(sp, &why) != MUON_OK) return fail(h, MUON_ERR_INVALID, "%s", why.c_str());
    }
    DeviceGuard dg(h->device);
    h->last_error.clear();
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    muon_status st = ensure_plan(h, shapes, s);
    if (st != MUON_OK) return st;
    if ((st = upload_segs(h, mp, s)) != MUON_OK) return st;
    return run_graph_or_direct(h, false, true, s, nullptr);
}

muon_status muon_ns_phase_run(muon_handle* h, const muon_ns_phase_args* a, void* stream) {
    if (!h) return MUON_ERR_INVALID;
    if (!a) return fail(h, MUON_ERR_INVALID, "args is NULL");
    if (a->phase < MUON_NS_GRAM || a->phase > MUON_NS_UPDATE) return fail(h, MUON_ERR_INVALID, "bad phase");
    if (a->precision != MUON_PREC_BF16 && a->precision != MUON_PREC_FP32_DEBUG) return fail(h, MUON_ERR_INVALID, "bad precision");
    std::string why;
    if (check_shape(a->m, a->n, a->count, &why) != MUON_OK) return fail(h, MUON_ERR_INVALID, "%s", why.c_str());
    if (!finite(a->alpha) || !finite(a->beta)) return fail(h, MUON_ERR_INVALID, "alpha and beta must be finite");
    if (!a->out) return fail(h, MUON_ERR_INVALID, "out is NULL");
    if (a->phase != MUON_NS_POLY && !a->x_op) return fail(h, MUON_ERR_INVALID, "x_op is NULL");
    if (a->phase != MUON_NS_GRAM && !a->a_in) return fail(h, MUON_ERR_INVALID, "a_in is NULL");
    if (a->phase == MUON_NS_UPDATE && !a->x_master) return fail(h, MUON_ERR_INVALID, "x_master is NULL");
    if (a->phase == MUON_NS_UPDATE && a->precision == MUON_PREC_BF16 && !a->out_op)
        return fail(h, MUON_ERR_INVALID, "out_op (low part of the result) is NULL");
    const bool bf16 = a->precision == MUON_PREC_BF16;
    if (bf16 && (a->m % 8 != 0 || a->n % 8 != 0)) return fail(h, MUON_ERR_UNSUPPORTED, "bf16 building blocks need m and n multiples of 8");
    const void* ptrs[5] = {a->x_op, a->a_in, a->x_master, a->out, a->out_op};
    for (const void* p : ptrs)
        if (p && !aligned(p, 16)) return fail(h, MUON_ERR_INVALID, "buffers must be 16-byte aligned");
    DeviceGuard dg(h->device);
    h->last_error.clear();
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int m = a->m, n = a->n, cnt = a->count;
    if (!bf16) {
        SimtGemmArgs g{};
        g.count = cnt;
        g.alpha = a->alpha; g.beta = a->beta;
        if (a->phase == MUON_NS_GRAM) {
            g.A = (const float*)a->x_op; g.B = (const float*)a->x_op; g.C = (float*)a->out;
            g.M = m; g.N = m; g.K = n; g.lda = n; g.ldb = n; g.ldc = m; g.sA = g.sB = (long long)m * n; g.sC = (long long)m * m; g.b_kmajor = 1;
        } else if (a->phase == MUON_NS_POLY) {
            g.A = (const float*)a->a_in; g.B = (const float*)a->a_in; g.C = (float*)a->out; g.Cin = (const float*)a->a_in;
            g.M = m; g.N = m; g.K = m; g.lda = g.ldb = g.ldc = g.ldcin = m; g.sA = g.sB = g.sC = g.sCin = (long long)m * m; g.b_kmajor = 1;
        } else {
            g.A = (const float*)a->a_in; g.B = (const float*)a->x_op; g.C = (float*)a->out;
            g.Cin = (const float*)a->x_master;
            g.M = m; g.N = n; g.K = m; g.lda = m; g.ldb = n; g.ldc = n; g.ldcin = n;
            g.sA = (long long)m * m; g.sB = g.sC = g.sCin = (long long)m * n; g.b_kmajor = 0;
        }
        CUDA_TRY(h, launch_simt_gemm(g, s));
        return MUON_OK;
    }
    muon_status st = load_encoder(h);
    if (st != MUON_OK) return st;
    if (!h->tc_ready) {
        CUDA_TRY(h, tc_gemm_prepare());
        CUDA_TRY(h, tc_gemm_max_clusters(&h->max_clusters));
        if (h->max_clusters < 1) return fail(h, MUON_ERR_UNSUPPORTED, "no two-CTA cluster fits on this device");
        h->tc_ready = true;
    }
    GroupDims d{};
    d.rows = m; d.cols = n; d.count = cnt; d.m = m; d.n = n; d.ldm = m; d.ldn = n; d.transposed = 0;
    std::vector<GroupDims> dims(1, d);
    const int phase = a->phase;
    std::vector<Tile> tl = build_tiles(dims, phase == MUON_NS_UPDATE ? 2 : phase, tc_gemm_tile_m(h->pair),
                                       tc_gemm_tile_n(h->pair));
    GemmMaps maps{};
    GemmGroupInfo gi{};
    gi.m = m; gi.n = n; gi.ldm = m; gi.ldn = n; gi.count = cnt; gi.mat_base = 0;
    if (phase == MUON_NS_GRAM) {
        if ((st = encode_map(h, &maps.xb_k[0], a->x_op, n, m, cnt, n, 128)) != MUON_OK) return st;
        if ((st = encode_sym_maps(h, maps.se_a, a->out, m, cnt, m)) != MUON_OK) return st;
        gi.a = (__nv_bfloat16*)a->out;
    } else if (phase == MUON_NS_POLY) {
        if ((st = encode_map(h, &maps.a, a->a_in, m, m, cnt, m, 128)) != MUON_OK) return st;
        if ((st = encode_sym_maps(h, maps.se_a, a->a_in, m, cnt, m)) != MUON_OK) return st;
        if ((st = encode_sym_maps(h, maps.se_p, a->out, m, cnt, m)) != MUON_OK) return st;
        gi.a = (__nv_bfloat16*)a->a_in;
        gi.p = (__nv_bfloat16*)a->out;
    } else {
        if ((st = encode_map(h, &maps.p, a->a_in, m, m, cnt, m, 128)) != MUON_OK) return st;
        if ((st = encode_map(h, &maps.xb_mn[0], a->x_op, n, m, cnt, n, 64)) != MUON_OK) return st;
        if ((st = encode_epi_map(h, &maps.xe_hi[0], a->x_op, n, m, cnt, n)) != MUON_OK) return st;
        if ((st = encode_epi_map(h, &maps.xe_hi[1], a->out, n, m, cnt, n)) != MUON_OK) return st;
        if ((st = encode_epi_map(h, &maps.xe_lo_in, a->x_master, n, m, cnt, n)) != MUON_OK) return st;
        if ((st = encode_epi_map(h, &maps.xe_lo_out, a->out_op, n, m, cnt, n)) != MUON_OK) return st;
        gi.xb[0] = (__nv_bfloat16*)a->x_op;            // X = x_op + x_master (high + low part)
        gi.xlo_in = (const __nv_bfloat16*)a->x_master;
        gi.xb[1] = (__nv_bfloat16*)a->out;              // X' = out + out_op
        gi.xlo_out = (__nv_bfloat16*)a->out_op;
    }
    // unit lists of the two-CTA kernel (split tiles included, so the building
    // blocks exercise the partial-sum path too)
    UnitPlan up;
    if (h->pair) {
        std::vector<int> kb;
        for (size_t i = 0; i < tl.size(); ++i) kb.push_back(((phase == MUON_NS_GRAM ? n : m) + TC_BK - 1) / TC_BK);
        up = build_units(tl, kb, h->max_clusters, tc_gemm_split_tiles() != 0, true);
    }
    std::vector<int4> uv;
    for (const Unit& u : up.units) {
        uv.push_back(make_int4(u.tile.group, u.tile.mat, u.tile.tile_row, u.tile.tile_col));
        uv.push_back(make_int4(u.k_begin, u.k_end, u.kind | (u.n_half << 8), u.slot | (u.nslots << 16)));
    }
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = align_up(off, 256); off = o + align_up(bytes, 256); return o; };
    const size_t o_maps = take(sizeof(GemmMaps)), o_gi = take(sizeof(GemmGroupInfo));
    const size_t o_t = take(tl.size() * sizeof(int4) + 16), o_u = take(uv.size() * sizeof(int4) + 16);
    const size_t o_ub = take(up.begin.size() * sizeof(int) + 16);
    const size_t o_skp = take((size_t)up.nslots * SK_SLOT_FLOATS * sizeof(float) + 16);
    const size_t o_skc = take((size_t)up.nslots * sizeof(int) + 16), o_skf = take((size_t)up.nslots * sizeof(int) + 16);
    // the scratch area may still be read by an earlier launch on another stream
    if (h->scratch.ptr) CUDA_TRY(h, cudaDeviceSynchronize());
    if ((st = ensure_buf(h, h->scratch, off)) != MUON_OK) return st;
    char* base = static_cast<char*>(h->scratch.ptr);
    std::vector<int4> tv(tl.size());
    for (size_t i = 0; i < tl.size(); ++i) tv[i] = make_int4(tl[i].group, tl[i].mat, tl[i].tile_row, tl[i].tile_col);
    CUDA_TRY(h, cudaMemcpyAsync(base + o_maps, &maps, sizeof(maps), cudaMemcpyHostToDevice, s));
    CUDA_TRY(h, cudaMemcpyAsync(base + o_gi, &gi, sizeof(gi), cudaMemcpyHostToDevice, s));
    CUDA_TRY(h, cudaMemcpyAsync(base + o_t, tv.data(), tv.size() * sizeof(int4), cudaMemcpyHostToDevice, s));
    if (!uv.empty()) CUDA_TRY(h, cudaMemcpyAsync(base + o_u, uv.data(), uv.size() * sizeof(int4), cudaMemcpyHostToDevice, s));
    if (!up.begin.empty())
        CUDA_TRY(h, cudaMemcpyAsync(base + o_ub, up.begin.data(), up.begin.size() * sizeof(int), cudaMemcpyHostToDevice, s));
    CUDA_TRY(h, cudaMemsetAsync(base + o_skc, 0, (size_t)up.nslots * sizeof(int) + 16, s));
    CUDA_TRY(h, cudaMemsetAsync(base + o_skf, 0, (size_t)up.nslots * sizeof(int) + 16, s));
    CUDA_TRY(h, cudaStreamSynchronize(s));
    GemmParams gp{};
    gp.units = reinterpret_cast<const int4*>(base + o_u);
    gp.unit_begin = reinterpret_cast<const int*>(base + o_ub);
    gp.sk_partial = reinterpret_cast<float*>(base + o_skp);
    gp.sk_count = reinterpret_cast<int*>(base + o_skc);
    gp.sk_flag = reinterpret_cast<int*>(base + o_skf);
    gp.epoch = 1;
    gp.tiles = reinterpret_cast<const int4*>(base + o_t);
    gp.ntiles = (int)tl.size();
    gp.maps = reinterpret_cast<const GemmMaps*>(base + o_maps);
    gp.groups = reinterpret_cast<const GemmGroupInfo*>(base + o_gi);
    gp.parity = 0;
    gp.alpha = a->alpha;
    gp.beta = a->beta;
    gp.scale = nullptr;
    gp.err = h->d_err;
    const int mode = phase == MUON_NS_GRAM ? MODE_GRAM : phase == MUON_NS_POLY ? MODE_POLY : MODE_UPDATE;
    CUDA_TRY(h, launch_tc_gemm(mode, h->pair, gp, gemm_grid(h, gp.ntiles, h->pair ? active_clusters(up, h->max_clusters) : 0),
                               s, tc_gemm_var(mode, phase == MUON_NS_GRAM ? n : m)));
    return MUON_OK;
}

muon_status muon_qk_clip(muon_handle* h, float* Wq, float* Wk, const float* max_logits, int n_heads, int head_dim,
                         int cols, float tau, void* stream) {
    if (!h) return MUON_ERR_INVALID;
    if (!Wq || !max_logits) return fail(h, MUON_ERR_INVALID, "Wq and max_logits are required");
    if (n_heads <= 0 || head_dim <= 0 || cols <= 0) return fail(h, MUON_ERR_INVALID, "sizes must be > 0");
    if ((long long)n_heads * head_dim * cols > (1ll << 31) - 1) return fail(h, MUON_ERR_INVALID, "matrix too large");
    if (!(finite(tau) && tau > 0.f)) return fail(h, MUON_ERR_INVALID, "tau must be finite and > 0");
    if (!aligned(Wq, 4) || (Wk && !aligned(Wk, 4)) || !aligned(max_logits, 4))
        return fail(h, MUON_ERR_INVALID, "misaligned pointer");
    DeviceGuard dg(h->device);
    h->last_error.clear();
    CUDA_TRY(h, launch_qk_clip(Wq, Wk, max_logits, n_heads, head_dim, cols, tau, h->num_sms,
                               static_cast<cudaStream_t>(stream)));
    return MUON_OK;
}

muon_status muon_sync(muon_handle* h, void* stream) {
    if (!h) return MUON_ERR_INVALID;
    DeviceGuard dg(h->device);
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(h, MUON_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
    int err = 0;
    CUDA_TRY(h, cudaMemcpy(&err, h->d_err, sizeof(int), cudaMemcpyDeviceToHost));
    if (err != 0) {
        CUDA_TRY(h, cudaMemset(h->d_err, 0, sizeof(int)));
        return fail(h, MUON_ERR_DEVICE_TIMEOUT, "a kernel gave up a bounded wait (code 0x%x)", err);
    }
    return MUON_OK;
}

muon_status muon_last_norms(muon_handle* h, float* out, int cap, int* n_out, void* stream) {
    if (!h || !n_out) return MUON_ERR_INVALID;
    if (!h->plan.valid) return fail(h, MUON_ERR_INVALID, "no step has run on this handle");
    *n_out = h->plan.nmat;
    if (!out || cap < h->plan.nmat) return fail(h, MUON_ERR_INVALID, "output holds %d floats, %d needed", cap, h->plan.nmat);
    DeviceGuard dg(h->device);
    CUDA_TRY(h, cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    CUDA_TRY(h, cudaMemcpy(out, h->plan.d_norms, h->plan.nmat * sizeof(float), cudaMemcpyDeviceToHost));
    return MUON_OK;
}

muon_status muon_last_update_rms(muon_handle* h, float* out, int cap, int* n_out, void* stream) {
    if (!h || !n_out) return MUON_ERR_INVALID;
    Plan& P = h->plan;
    if (!P.valid || P.uploaded.empty()) return fail(h, MUON_ERR_INVALID, "no step has run on this handle");
    *n_out = P.nmat;
    if (!out || cap < P.nmat) return fail(h, MUON_ERR_INVALID, "output holds %d floats, %d needed", cap, P.nmat);
    DeviceGuard dg(h->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CUDA_TRY(h, launch_update_rms(P.d_segs, P.nmat, h->cfg.ns_steps == 0 ? P.d_scale : nullptr, h->cfg.lr,
                                  P.d_rms_part, P.d_rms, s));
    CUDA_TRY(h, cudaStreamSynchronize(s));
    CUDA_TRY(h, cudaMemcpy(out, P.d_rms, P.nmat * sizeof(float), cudaMemcpyDeviceToHost));
    return MUON_OK;
}

muon_status muon_last_update(muon_handle* h, int group, int index, float* dst, void* stream) {
    if (!h || !dst) return MUON_ERR_INVALID;
    Plan& P = h->plan;
    if (!P.valid || P.uploaded.empty()) return fail(h, MUON_ERR_INVALID, "no step has run on this handle");
    if (group < 0 || group >= (int)P.dims.size() || index < 0 || index >= P.dims[group].count)
        return fail(h, MUON_ERR_INVALID, "no matrix %d in group %d", index, group);
    DeviceGuard dg(h->device);
    const EwSeg& sg = P.uploaded[P.mat_base[group] + index];
    CUDA_TRY(h, launch_copy_out_one(sg, dst, h->cfg.ns_steps == 0 ? P.d_scale : nullptr, static_cast<cudaStream_t>(stream)));
    return MUON_OK;
}

muon_status muon_timing_enable(muon_handle* h, int enable) {
    if (!h) return MUON_ERR_INVALID;
    h->timing = enable != 0;
    return MUON_OK;
}

muon_status muon_timing_read(muon_handle* h, double* ms, int* launches, int n_kinds, void* stream) {
    if (!h || n_kinds < 0 || n_kinds > MUON_TIMING_KINDS) return MUON_ERR_INVALID;
    DeviceGuard dg(h->device);
    CUDA_TRY(h, cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    for (const auto& p : h->pending) {
        float t = 0.f;
        CUDA_TRY(h, cudaEventSynchronize(p.b));
        CUDA_TRY(h, cudaEventElapsedTime(&t, p.a, p.b));
        h->t_ms[p.kind] += t;
        h->t_n[p.kind] += 1;
        h->ev_free.push_back(p.a);
        h->ev_free.push_back(p.b);
    }
    h->pending.clear();
    for (int k = 0; k < n_kinds; ++k) {
        if (ms) ms[k] = h->t_ms[k];
        if (launches) launches[k] = h->t_n[k];
    }
    for (int k = 0; k < MUON_TIMING_KINDS; ++k) { h->t_ms[k] = 0.0; h->t_n[k] = 0; }
    return MUON_OK;
}

muon_status muon_destroy(muon_handle* h) {
    if (!h) return MUON_ERR_INVALID;
    {
        DeviceGuard dg(h->device);
        cudaDeviceSynchronize();
        for (auto& p : h->pending) { cudaEventDestroy(p.a); cudaEventDestroy(p.b); }
        for (auto e : h->ev_free) cudaEventDestroy(e);
        cudaEvent_t evs[4] = {h->ev_start, h->ev_w, h->ev_k1, h->ev_done};
        for (cudaEvent_t e : evs) if (e) cudaEventDestroy(e);
        if (h->side) cudaStreamDestroy(h->side);
        if (h->side2) cudaStreamDestroy(h->side2);
        if (h->gexec) cudaGraphExecDestroy(h->gexec);
        if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
        if (h->ws.ptr) cudaFree(h->ws.ptr);
        if (h->staging.ptr) cudaFree(h->staging.ptr);
        if (h->scratch.ptr) cudaFree(h->scratch.ptr);
        if (h->apply_segs.ptr) cudaFree(h->apply_segs.ptr);
        if (h->d_err) cudaFree(h->d_err);
    }
    delete h;
    return MUON_OK;
}

const char* muon_last_error(const muon_handle* h) { return h ? h->last_error.c_str() : "NULL handle"; }

const char* muon_status_string(muon_status s) {
    switch (s) {
        case MUON_OK: return "MUON_OK";
        case MUON_ERR_INVALID: return "MUON_ERR_INVALID";
        case MUON_ERR_UNSUPPORTED: return "MUON_ERR_UNSUPPORTED";
        case MUON_ERR_OOM: return "MUON_ERR_OOM";
        case MUON_ERR_CUDA: return "MUON_ERR_CUDA";
        case MUON_ERR_DEVICE_TIMEOUT: return "MUON_ERR_DEVICE_TIMEOUT";
    }
    return "unknown status";
}

int muon_plan_tile_m(void) { return tc_gemm_tile_m(tc_gemm_default_pair()); }
int muon_plan_tile_n(void) { return tc_gemm_tile_n(tc_gemm_default_pair()); }

muon_status muon_plan_tiles(const int* shapes, int n_groups, int phase, int* out, int cap, int* n_tiles) {
    if (!shapes || n_groups <= 0 || !n_tiles || phase < 0 || phase > 2) return MUON_ERR_INVALID;
    std::vector<GroupDims> dims;
    for (int g = 0; g < n_groups; ++g) {
        std::string why;
        if (check_shape(shapes[3 * g], shapes[3 * g + 1], shapes[3 * g + 2], &why) != MUON_OK) return MUON_ERR_INVALID;
        dims.push_back(make_dims(shapes[3 * g], shapes[3 * g + 1], shapes[3 * g + 2]));
    }
    const int pair = tc_gemm_default_pair();
    std::vector<Tile> t = build_tiles(dims, phase, tc_gemm_tile_m(pair), tc_gemm_tile_n(pair));
    std::vector<int> kb;
    for (const Tile& x : t) kb.push_back(((phase == 0 ? dims[x.group].n : dims[x.group].m) + TC_BK - 1) / TC_BK);
    if (!check_plan(dims, phase, tc_gemm_tile_m(pair), tc_gemm_tile_n(pair), TC_BK, t, kb, nullptr, 1).empty())
        return MUON_ERR_INVALID;
    *n_tiles = (int)t.size();
    if (!out || cap < (int)t.size()) return MUON_ERR_INVALID;
    for (size_t i = 0; i < t.size(); ++i) {
        out[4 * i] = t[i].group; out[4 * i + 1] = t[i].mat; out[4 * i + 2] = t[i].tile_row; out[4 * i + 3] = t[i].tile_col;
    }
    return MUON_OK;
}

muon_status muon_plan_units(const int* shapes, int n_groups, int phase, int clusters, int split, int* out,
                            int cap, int* n_units) {
    if (!shapes || n_groups <= 0 || !n_units || phase < 0 || phase > 2 || clusters < 1) return MUON_ERR_INVALID;
    std::vector<GroupDims> dims;
    for (int g = 0; g < n_groups; ++g) {
        std::string why;
        if (check_shape(shapes[3 * g], shapes[3 * g + 1], shapes[3 * g + 2], &why) != MUON_OK) return MUON_ERR_INVALID;
        dims.push_back(make_dims(shapes[3 * g], shapes[3 * g + 1], shapes[3 * g + 2]));
    }
    std::vector<Tile> t = build_tiles(dims, phase, tc_gemm_tile_m(1), tc_gemm_tile_n(1));
    std::vector<int> kb;
    for (const Tile& x : t) kb.push_back(((phase == 0 ? dims[x.group].n : dims[x.group].m) + TC_BK - 1) / TC_BK);
    UnitPlan up = build_units(t, kb, clusters, split != 0, split == 0);
    if (!check_plan(dims, phase, tc_gemm_tile_m(1), tc_gemm_tile_n(1), TC_BK, t, kb, &up, clusters).empty())
        return MUON_ERR_INVALID;
    *n_units = (int)up.units.size();
    if (!out || cap < (int)up.units.size()) return MUON_ERR_INVALID;
    for (int c = 0; c < clusters; ++c) {
        for (int i = up.begin[c]; i < up.begin[c + 1]; ++i) {
            const Unit& u = up.units[i];
            int* o = out + 11 * i;
            o[0] = c; o[1] = u.tile.group; o[2] = u.tile.mat; o[3] = u.tile.tile_row; o[4] = u.tile.tile_col;
            o[5] = u.k_begin; o[6] = u.k_end; o[7] = u.kind; o[8] = u.slot; o[9] = u.nslots; o[10] = u.n_half;
        }
    }
    return MUON_OK;
}

}  // extern "C"
