// C ABI of the library (declared in include/moefp8.h): argument checks,
// tile selection, workspace carving and the launch sequence of the fused
// layer.  No entry point allocates device memory.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <utility>
#include <vector>

#include "moefp8.h"
#include "common.cuh"
#include "kernels.h"

using namespace moe;

static_assert(MOE_MAX_EXPERTS == kMaxRouteExperts, "routing kernels and the C ABI disagree on E");

namespace {

// Status word for the entry points that take no workspace.
__device__ int g_lib_status[kStatusInts];

std::atomic<unsigned long long> g_timeout_ns{2000000000ull};
std::atomic<int> g_fusion{MOE_FUSION_AUTO};

constexpr int kStageEvents = 6;
cudaEvent_t g_stage_events[kStageEvents];
std::atomic<bool> g_stage_events_on{false};

inline void stage_mark(int i, cudaStream_t s) {
    if (g_stage_events_on.load(std::memory_order_relaxed) && g_stage_events[i])
        cudaEventRecord(g_stage_events[i], s);
}

struct DevInfo {
    int sms = 0;
    int major = 0, minor = 0;
    int* lib_status = nullptr;
    bool ok = false;
};

constexpr int kMaxDevices = 64;
DevInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Per-device facts, looked up once per device with that device current.
const DevInfo* dev_info() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo& d = g_dev[dev];
    if (!d.ok) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return nullptr;
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev);
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_lib_status) != cudaSuccess) return nullptr;
        d.lib_status = static_cast<int*>(p);
        d.ok = true;
    }
    return &d;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace of the fused layer, in carve order.
struct FusedWs {
    size_t status, m_indptr, chunk_hist, perm, inv_perm, xq, xs, hq, hs, out_acc, total;
};

FusedWs fused_layout(int T, int H, int I, int E, int k) {
    const size_t R = static_cast<size_t>(T) * k;
    const size_t nchunks = (R + kRouteChunk - 1) / kRouteChunk;
    FusedWs w{};
    size_t o = 0;
    w.status = o;     o += up256(sizeof(int) * kStatusInts);
    w.m_indptr = o;   o += up256(sizeof(int32_t) * (E + 1));
    w.chunk_hist = o; o += up256(sizeof(int32_t) * nchunks * E);
    w.perm = o;       o += up256(sizeof(int32_t) * R);
    w.inv_perm = o;   o += up256(sizeof(int32_t) * R);
    w.xq = o;         o += up256(R * H);
    w.xs = o;         o += up256(sizeof(float) * R * (H / 128));
    w.hq = o;         o += up256(R * I);
    w.hs = o;         o += up256(sizeof(float) * R * (I / 128));
    // FP8 layer: y [R, H] fp32, one row per pair (GEMM2's output); MXFP8 and
    // NVFP4 layers: their fp32 combine buffer [T, H] at the same place
    w.out_acc = o;    o += up256(sizeof(float) * R * H);
    w.total = o;
    return w;
}

size_t route_ws_bytes(int T, int k, int E) {
    const size_t R = static_cast<size_t>(T) * k;
    const size_t nchunks = (R + kRouteChunk - 1) / kRouteChunk;
    return up256(sizeof(int) * kStatusInts) + up256(sizeof(int32_t) * nchunks * E);
}

// --- tile selection (wave + residue), sm_100a tile menu -----------------
// Token tiles of 16/32/64 rows run with the weights as the 128-row MMA
// operand; 128-row tiles with the tokens as the MMA M operand.  Each tile
// covers 256 weight rows: 128 output columns gated, 256 plain.
constexpr int kTileOverheadRows = 32;

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }

long long balanced_tile_count(long long total_rows, long long n_out, long long E, int tile_m,
                              int tile_n) {
    const long long q = total_rows / E, r = total_rows % E;
    const long long m_tiles = r * ceil_div(q + 1, tile_m) + (E - r) * ceil_div(q, tile_m);
    return m_tiles * ceil_div(n_out, tile_n);
}

void select_tile(int total_rows, int n, int k, int E, int num_sms, int gated, int* tm, int* tn) {
    const long long n_out = gated ? n / 2 : n;
    const int tile_n = gated ? 128 : 256;
    *tn = tile_n;
    if (E <= 0 || total_rows <= 0) { *tm = 16; return; }
    const long long max_m = ceil_div(total_rows, E);
    auto tiles = [&](int t) { return balanced_tile_count(total_rows, n_out, E, t, tile_n); };
    if (max_m <= 16 || (tiles(32) < num_sms / 2 && tiles(16) <= num_sms)) { *tm = 16; return; }
    if (max_m <= 32) { *tm = 32; return; }
    if (k <= 2048) { *tm = max_m < 192 ? 64 : 128; return; }
    auto cost = [&](int t) { return ceil_div(tiles(t), num_sms) * (t + kTileOverheadRows); };
    *tm = cost(64) < cost(128) ? 64 : 128;
}

// --- tactic table: measured tile choice per GEMM shape class ---------------
// The cuTile page tunes each GEMM of the pair per architecture and shape
// ("2. cuTile NVFP4 양자화 지원"); here a process-wide table maps a shape class
// to the token tile that timed fastest on this GPU (moe_tactic_tune_gemm).
// Class: (N, K, E, gated, bucket of ceil(R / E)), the bucket being the power
// of two at or above the balanced rows per expert (8 or fewer -> 0).
struct TacticKey {
    int n, k, e, gated, bucket;
    bool operator==(const TacticKey& o) const {
        return n == o.n && k == o.k && e == o.e && gated == o.gated && bucket == o.bucket;
    }
};

int rows_bucket(long long R, int E) {
    const long long m = (R + E - 1) / E;
    int b = 0;
    for (long long v = 8; v < m && b < 24; v <<= 1) ++b;
    return b;
}

std::mutex g_tactic_mu;
std::vector<std::pair<TacticKey, int>> g_tactics;

bool tactic_lookup(const TacticKey& key, int* tm) {
    std::lock_guard<std::mutex> lk(g_tactic_mu);
    for (const auto& kv : g_tactics)
        if (kv.first == key) { *tm = kv.second; return true; }
    return false;
}

void tactic_store(const TacticKey& key, int tm) {
    std::lock_guard<std::mutex> lk(g_tactic_mu);
    for (auto& kv : g_tactics)
        if (kv.first == key) { kv.second = tm; return; }
    g_tactics.emplace_back(key, tm);
}

bool valid_tile_m(int tm) { return tm == 16 || tm == 32 || tm == 64 || tm == 128; }

// tile_m for a GEMM launched with tile_m = -1: the tuned entry of its shape
// class when there is one, else the wave + residue model.
int choose_tile_m(int R, int N, int K, int E, int gated, int num_sms) {
    int tm, tn;
    if (!tactic_lookup(TacticKey{N, K, E, gated ? 1 : 0, rows_bucket(R, E)}, &tm))
        select_tile(R, N, K, E, num_sms, gated ? 1 : 0, &tm, &tn);
    return tm;
}

// Token tiles of the swapped kernels stage K/128 x tile_m scales on chip.
int fit_tile_to_k(int tm, int K) {
    while (tm < 128 && K > swap_max_k(tm)) tm *= 2;
    return tm;
}

// The fused-expert launch runs each (expert, 64-token group) on one SM,
// streaming that expert's weights through one SM's share of the memory
// system (the groups of one expert run side by side and share its weights
// through L2); the split GEMMs spread every expert's weights over many SMs.
// Measured on B200 (whole layer, µs, fused / split, top-8): H=2048 I=768
// E=128 at T=512: 160 / 213, at T=2048: 385 / 496; T=1024 H=1024 I=512
// E=160: 135 / 152; T=16 H=256 I=128 E=4: 31 / 34.  A second round of
// experts (T=64 E=256: 253 / 213), half the SMs idle (E=64, top-4:
// 287 / 263) or 12.6 MB experts (H=4096 I=1024: 308 / 296) lose.  So: tiny
// layers (one launch fewer), else about one round of active experts filling
// at least half the SMs, at most ~2 rounds of groups, experts of <= 6 MB.
bool fuse_pays(int R, int H, int I, int E, int num_sms) {
    const long long per = (static_cast<long long>(R) + E - 1) / E;   // rows per expert, balanced
    const long long active = R < E ? R : E;
    const long long items = active * ((per + 63) / 64);
    const long long expert_bytes = 3LL * H * I;
    if (active * expert_bytes <= (16LL << 20)) return true;
    return active <= num_sms + num_sms / 8 && 2 * active >= num_sms &&
           items <= 2 * num_sms + num_sms / 4 && expert_bytes <= 6000000LL;
}

// Launch plan of the FP8 fused layer: GEMM1 / GEMM2 token tiles and whether
// both GEMMs run as one fused-expert launch.
struct LayerPlan {
    int tm1, tm2;
    bool fuse;
};

LayerPlan plan_layer(int R, int H, int I, int E, int num_sms) {
    LayerPlan pl;
    pl.tm1 = fit_tile_to_k(choose_tile_m(R, 2 * I, H, E, 1, num_sms), H);
    pl.tm2 = fit_tile_to_k(choose_tile_m(R, H, I, E, 0, num_sms), I);
    const int fmode = g_fusion.load();
    pl.fuse = fmode != MOE_FUSION_OFF && fused_expert_fits(H, I, E) &&
              (fmode == MOE_FUSION_ON || (pl.tm1 < 128 && fuse_pays(R, H, I, E, num_sms)));
    return pl;
}

int check_device(const DevInfo* d) {
    if (!d) return MOE_ERR_CUDA;
    if (d->major != 10 || d->minor != 0) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_NO_TILE_CONFIG: return "MOE_ERR_NO_TILE_CONFIG";
        case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
        case MOE_ERR_BAD_EXPERT_ID: return "MOE_ERR_BAD_EXPERT_ID";
        default: return "MOE_ERR_UNKNOWN";
    }
}

void moe_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns > 0 ? ns : 1); }

int moe_fp8_fused_plan(int T, int H, int I, int E, int k, int* tile_m1, int* tile_m2,
                       int* fused) {
    if (T < 0 || H <= 0 || I <= 0 || H % 128 || I % 128 || k < 1 || E < 1 || k > E)
        return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    const LayerPlan pl = plan_layer(T * k, H, I, E, d->sms);
    if (tile_m1) *tile_m1 = pl.tm1;
    if (tile_m2) *tile_m2 = pl.tm2;
    if (fused) *fused = pl.fuse ? 1 : 0;
    return MOE_OK;
}

int moe_set_expert_fusion(int mode) {
    if (mode != MOE_FUSION_AUTO && mode != MOE_FUSION_ON && mode != MOE_FUSION_OFF)
        return MOE_ERR_INVALID_ARG;
    g_fusion.store(mode);
    return MOE_OK;
}

int moe_set_stage_events(void* const* events, int n) {
    if (events == nullptr) {
        g_stage_events_on.store(false);
        return MOE_OK;
    }
    if (n != kStageEvents) return MOE_ERR_INVALID_ARG;
    bool any = false;
    for (int i = 0; i < kStageEvents; ++i) any = any || events[i] != nullptr;
    if (!any) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < kStageEvents; ++i) g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_stage_events_on.store(true);
    return MOE_OK;
}

int moe_select_tile_m(int total_rows, int n, int k, int E, int num_sms, int is_gated, int* tile_m,
                      int* tile_n) {
    if (!tile_m || !tile_n || num_sms <= 0 || total_rows < 0 || n <= 0 || k <= 0 || E <= 0)
        return MOE_ERR_INVALID_ARG;
    select_tile(total_rows, n, k, E, num_sms, is_gated ? 1 : 0, tile_m, tile_n);
    return MOE_OK;
}

size_t moe_route_workspace_size(int T, int k, int E) {
    if (T < 0 || k < 1 || E < 1) return 0;
    return route_ws_bytes(T, k, E);
}

int moe_route_permute(const int32_t* topk_ids, int T, int k, int E, int32_t* m_indptr,
                      int32_t* perm, int32_t* inv_perm, void* ws, size_t ws_bytes,
                      moe_stream_t stream) {
    if (T < 0 || k < 1 || E < 1 || E > MOE_MAX_EXPERTS) return MOE_ERR_INVALID_ARG;
    if (!m_indptr || !ws || (T > 0 && (!topk_ids || !perm))) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < route_ws_bytes(T, k, E) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* base = static_cast<char*>(ws);
    int* status = reinterpret_cast<int*>(base);
    if (cudaMemsetAsync(status, 0, sizeof(int) * kStatusInts, s) != cudaSuccess) return MOE_ERR_CUDA;
    RouteArgs ra{topk_ids, T, k, E, m_indptr, perm, inv_perm,
                 reinterpret_cast<int32_t*>(base + up256(sizeof(int) * kStatusInts)), status};
    return launch_route_permute(ra, s);
}

size_t moe_workspace_size(int T, int H, int I, int E, int k) {
    if (T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1) return 0;
    return fused_layout(T, H, I, E, k).total;
}

static int fused_impl(const void* x, const int32_t* topk_ids, const float* topk_w, const void* w13,
                      const float* w13_scale, const void* w2, const float* w2_scale, void* out, int T,
                      int H, int I, int E, int k, void* ws, size_t ws_bytes, moe_stream_t stream,
                      int32_t* dbg_m_indptr, int32_t* dbg_perm, uint8_t* dbg_hq, float* dbg_hs) {
    if (T < 0 || H <= 0 || I <= 0 || H % 128 || I % 128 || k < 1) return MOE_ERR_INVALID_ARG;
    if (E < 1) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (k > E) return MOE_ERR_INVALID_ARG;
    if (!ws) return MOE_ERR_INVALID_ARG;
    const FusedWs L = fused_layout(T, H, I, E, k);
    if (ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    if (T > 0) {
        if (!x || !topk_ids || !topk_w || !w13 || !w13_scale || !w2 || !w2_scale || !out)
            return MOE_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(w13) || !aligned16(w2) || !aligned16(out))
            return MOE_ERR_INVALID_ARG;
    }
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    int* status = reinterpret_cast<int*>(b + L.status);
    int32_t* m_indptr = reinterpret_cast<int32_t*>(b + L.m_indptr);
    int32_t* perm = reinterpret_cast<int32_t*>(b + L.perm);
    int32_t* inv_perm = reinterpret_cast<int32_t*>(b + L.inv_perm);
    uint8_t* xq = reinterpret_cast<uint8_t*>(b + L.xq);
    float* xs = reinterpret_cast<float*>(b + L.xs);
    uint8_t* hq = reinterpret_cast<uint8_t*>(b + L.hq);
    float* hs = reinterpret_cast<float*>(b + L.hs);
    float* out_acc = reinterpret_cast<float*>(b + L.out_acc);
    const int R = T * k;
    // the single-launch routing kernel clears the status words itself
    const bool route_clears = route_single_launch(R);
    if (!route_clears && cudaMemsetAsync(status, 0, sizeof(int) * kStatusInts, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    RouteArgs ra{topk_ids, T, k, E, m_indptr, perm, inv_perm,
                 reinterpret_cast<int32_t*>(b + L.chunk_hist), status, route_clears ? 1 : 0};
    stage_mark(0, s);
    int st = launch_route_permute(ra, s);
    if (st) return st;
    stage_mark(1, s);
    if (T > 0) {
        const LayerPlan pl = plan_layer(R, H, I, E, d->sms);
        const int tm1 = pl.tm1, tm2 = pl.tm2;
        // Swapped (small-group) GEMM1 tiles gather each grouped row's token
        // row through perm (TMA gather4), so x is quantised once per token
        // ([T, H], scales [H/128, T]).  128-token tiles load their rows as
        // two tiled boxes per K block, which gathered rows cannot match, so
        // there the quantiser writes the k grouped copies ([R, H], [H/128, R]).
        // The fused-expert launch reads the grouped copies too (one tiled box
        // of 64 rows per K block).
        const bool fuse = pl.fuse;
        const bool gather = tm1 < 128 && !fuse;
        const bool per_token = gather;
        st = per_token ? launch_quant_scatter(x, T, H, 1, T, nullptr, xq, xs, nullptr, s)
                       : launch_quant_scatter(x, T, H, k, R, inv_perm, xq, xs, nullptr, s);
        if (st) return st;
        stage_mark(2, s);
        const unsigned long long tmo = g_timeout_ns.load();
        float* y = out_acc;
        if (fuse) {
            FusedExpertArgs f{};
            f.xq = xq; f.xs = xs; f.R = R; f.H = H; f.I = I;
            f.E = E; f.w13 = w13; f.w13_scale = w13_scale; f.w2 = w2; f.w2_scale = w2_scale;
            f.m_indptr = m_indptr; f.y = y;
            // the intermediate leaves the chip only for the debug outputs
            f.hq = dbg_hq ? hq : nullptr;
            f.hs = dbg_hs ? hs : nullptr;
            f.status = status; f.timeout_ns = tmo; f.num_sms = d->sms;
            st = launch_fused_expert(f, s);
            if (st) return st;
            stage_mark(3, s);
            stage_mark(4, s);
            st = launch_combine(y, inv_perm, topk_w, T, k, H, out, s);
            if (st) return st;
            stage_mark(5, s);
        } else {
        GemmArgs g1{};
        g1.a = xq; g1.b = w13; g1.R = R; g1.N = 2 * I; g1.K = H; g1.E = E;
        g1.a_scale = xs; g1.as_row = 1; g1.as_kb = gather ? T : R; g1.b_scale = w13_scale;
        if (gather) { g1.a_rowmap = perm; g1.a_rowdiv = k; g1.a_rows = T; }
        g1.m_indptr = m_indptr; g1.epi = EPI_SWIGLU_QUANT; g1.tile_m = tm1;
        g1.hq = hq; g1.hs = hs; g1.status = status; g1.timeout_ns = tmo; g1.num_sms = d->sms;
        st = launch_grouped_gemm(g1, s);
        if (st) return st;
        stage_mark(3, s);
        // GEMM2 writes each pair's row y once, in grouped order; the combine
        // then sums each token's k rows in ascending slot order
        GemmArgs g2{};
        g2.a = hq; g2.b = w2; g2.R = R; g2.N = H; g2.K = I; g2.E = E;
        g2.a_scale = hs; g2.as_row = 1; g2.as_kb = R; g2.b_scale = w2_scale;
        g2.m_indptr = m_indptr; g2.epi = EPI_Y32; g2.tile_m = tm2;
        g2.y = y; g2.ldy = H;
        g2.status = status; g2.timeout_ns = tmo; g2.num_sms = d->sms;
        st = launch_grouped_gemm(g2, s);
        if (st) return st;
        stage_mark(4, s);
        st = launch_combine(y, inv_perm, topk_w, T, k, H, out, s);
        if (st) return st;
        stage_mark(5, s);
        }
    }
    if (dbg_m_indptr &&
        cudaMemcpyAsync(dbg_m_indptr, m_indptr, sizeof(int32_t) * (E + 1), cudaMemcpyDeviceToDevice, s))
        return MOE_ERR_CUDA;
    if (R > 0) {
        if (dbg_perm &&
            cudaMemcpyAsync(dbg_perm, perm, sizeof(int32_t) * R, cudaMemcpyDeviceToDevice, s))
            return MOE_ERR_CUDA;
        if (dbg_hq &&
            cudaMemcpyAsync(dbg_hq, hq, static_cast<size_t>(R) * I, cudaMemcpyDeviceToDevice, s))
            return MOE_ERR_CUDA;
        if (dbg_hs && cudaMemcpyAsync(dbg_hs, hs, sizeof(float) * static_cast<size_t>(R) * (I / 128),
                                      cudaMemcpyDeviceToDevice, s))
            return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

// The fused layer with MXFP8 operands.  Same workspace layout as the FP8
// path: the fp32 scale regions (4 bytes per 128 columns per row) hold the
// E8M0 scales (one byte per 32 columns per row) in [K/128, R, 4] order.
static int mx_fused_impl(const void* x, const int32_t* topk_ids, const float* topk_w,
                         const void* w13, const uint8_t* w13_sf, const void* w2,
                         const uint8_t* w2_sf, void* out, int T, int H, int I, int E, int k,
                         void* ws, size_t ws_bytes, moe_stream_t stream, int32_t* dbg_m_indptr,
                         int32_t* dbg_perm, uint8_t* dbg_hq, uint8_t* dbg_hsf) {
    if (T < 0 || H <= 0 || I <= 0 || H % 128 || I % 128 || k < 1) return MOE_ERR_INVALID_ARG;
    if (E < 1) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (k > E) return MOE_ERR_INVALID_ARG;
    if (!ws) return MOE_ERR_INVALID_ARG;
    const FusedWs L = fused_layout(T, H, I, E, k);
    if (ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    if (T > 0) {
        if (!x || !topk_ids || !topk_w || !w13 || !w13_sf || !w2 || !w2_sf || !out)
            return MOE_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(w13) || !aligned16(w2) || !aligned16(out) ||
            !aligned16(w13_sf) || !aligned16(w2_sf))
            return MOE_ERR_INVALID_ARG;
    }
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    int* status = reinterpret_cast<int*>(b + L.status);
    int32_t* m_indptr = reinterpret_cast<int32_t*>(b + L.m_indptr);
    int32_t* perm = reinterpret_cast<int32_t*>(b + L.perm);
    int32_t* inv_perm = reinterpret_cast<int32_t*>(b + L.inv_perm);
    uint8_t* xq = reinterpret_cast<uint8_t*>(b + L.xq);
    uint8_t* xsf = reinterpret_cast<uint8_t*>(b + L.xs);
    uint8_t* hq = reinterpret_cast<uint8_t*>(b + L.hq);
    uint8_t* hsf = reinterpret_cast<uint8_t*>(b + L.hs);
    float* out_acc = reinterpret_cast<float*>(b + L.out_acc);
    if (cudaMemsetAsync(status, 0, sizeof(int) * kStatusInts, s) != cudaSuccess) return MOE_ERR_CUDA;
    const int R = T * k;
    RouteArgs ra{topk_ids, T, k, E, m_indptr, perm, inv_perm,
                 reinterpret_cast<int32_t*>(b + L.chunk_hist), status};
    stage_mark(0, s);
    int st = launch_route_permute(ra, s);
    if (st) return st;
    stage_mark(1, s);
    if (T > 0) {
        st = launch_mx_quant_scatter(x, T, H, k, R, inv_perm, xq, xsf, out_acc, s);
        if (st) return st;
        stage_mark(2, s);
        const unsigned long long tmo = g_timeout_ns.load();
        MxGemmArgs g1{};
        g1.a = xq; g1.b = w13; g1.a_sf = xsf; g1.a_sf_mn = 1; g1.b_sf = w13_sf;
        g1.m_indptr = m_indptr; g1.R = R; g1.N = 2 * I; g1.K = H; g1.E = E; g1.gated = 1;
        g1.epi = MX_EPI_SWIGLU_MXQUANT; g1.hq = hq; g1.hsf = hsf;
        g1.status = status; g1.timeout_ns = tmo; g1.num_sms = d->sms;
        st = launch_mx_gemm(g1, s);
        if (st) return st;
        stage_mark(3, s);
        MxGemmArgs g2{};
        g2.a = hq; g2.b = w2; g2.a_sf = hsf; g2.a_sf_mn = 1; g2.b_sf = w2_sf;
        g2.m_indptr = m_indptr; g2.R = R; g2.N = H; g2.K = I; g2.E = E; g2.gated = 0;
        g2.epi = MX_EPI_COMBINE; g2.perm = perm; g2.topk_w = topk_w; g2.topk = k;
        g2.out_acc = out_acc; g2.out_ld = H;
        g2.status = status; g2.timeout_ns = tmo; g2.num_sms = d->sms;
        st = launch_mx_gemm(g2, s);
        if (st) return st;
        stage_mark(4, s);
        st = launch_f32_to_bf16(out_acc, out, static_cast<long long>(T) * H, d->sms, s);
        if (st) return st;
        stage_mark(5, s);
    }
    if (dbg_m_indptr &&
        cudaMemcpyAsync(dbg_m_indptr, m_indptr, sizeof(int32_t) * (E + 1), cudaMemcpyDeviceToDevice, s))
        return MOE_ERR_CUDA;
    if (R > 0) {
        if (dbg_perm &&
            cudaMemcpyAsync(dbg_perm, perm, sizeof(int32_t) * R, cudaMemcpyDeviceToDevice, s))
            return MOE_ERR_CUDA;
        if (dbg_hq &&
            cudaMemcpyAsync(dbg_hq, hq, static_cast<size_t>(R) * I, cudaMemcpyDeviceToDevice, s))
            return MOE_ERR_CUDA;
        if (dbg_hsf &&
            cudaMemcpyAsync(dbg_hsf, hsf, static_cast<size_t>(R) * (I / 32), cudaMemcpyDeviceToDevice, s))
            return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

int moe_mxfp8_fused(const void* x, const int32_t* topk_ids, const float* topk_w, const void* w13,
                    const uint8_t* w13_sf, const void* w2, const uint8_t* w2_sf, void* out, int T,
                    int H, int I, int E, int k, void* ws, size_t ws_bytes, moe_stream_t stream) {
    return mx_fused_impl(x, topk_ids, topk_w, w13, w13_sf, w2, w2_sf, out, T, H, I, E, k, ws,
                         ws_bytes, stream, nullptr, nullptr, nullptr, nullptr);
}

int moe_mxfp8_fused_debug(const void* x, const int32_t* topk_ids, const float* topk_w,
                          const void* w13, const uint8_t* w13_sf, const void* w2,
                          const uint8_t* w2_sf, void* out, int T, int H, int I, int E, int k,
                          void* ws, size_t ws_bytes, moe_stream_t stream, int32_t* m_indptr,
                          int32_t* perm, uint8_t* h_fp8, uint8_t* h_sf) {
    return mx_fused_impl(x, topk_ids, topk_w, w13, w13_sf, w2, w2_sf, out, T, H, I, E, k, ws,
                         ws_bytes, stream, m_indptr, perm, h_fp8, h_sf);
}

// The fused layer in the NVFP4 variant.  Workspace: the layout of the FP8
// layer; packed codes and their E4M3 scales (9/16 of the FP8 code bytes) sit
// in the code regions, codes first.
static int nv_fused_impl(const void* x, const int32_t* topk_ids, const float* topk_w,
                         const void* w13, const uint8_t* w13_sf, const float* w13_alpha,
                         const void* w2, const uint8_t* w2_sf, const float* w2_alpha,
                         float a1_gscale, float a2_gscale, void* out, int T, int H, int I, int E,
                         int k, void* ws, size_t ws_bytes, moe_stream_t stream,
                         int32_t* dbg_m_indptr, int32_t* dbg_perm, uint8_t* dbg_hq,
                         uint8_t* dbg_hsf) {
    if (T < 0 || H <= 0 || I <= 0 || H % 256 || I % 256 || k < 1) return MOE_ERR_INVALID_ARG;
    if (E < 1) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (k > E) return MOE_ERR_INVALID_ARG;
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (!(a1_gscale > 0.0f) || !(a2_gscale > 0.0f)) return MOE_ERR_INVALID_ARG;
    const FusedWs L = fused_layout(T, H, I, E, k);
    if (ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    if (T > 0) {
        if (!x || !topk_ids || !topk_w || !w13 || !w13_sf || !w13_alpha || !w2 || !w2_sf ||
            !w2_alpha || !out)
            return MOE_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(w13) || !aligned16(w2) || !aligned16(out) ||
            !aligned16(w13_sf) || !aligned16(w2_sf))
            return MOE_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(w13_alpha) | reinterpret_cast<uintptr_t>(w2_alpha)) & 3)
            return MOE_ERR_INVALID_ARG;
    }
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    const size_t R = static_cast<size_t>(T) * k;
    const size_t xsf_off = L.xq + up256(R * H / 2);
    const size_t hsf_off = L.hq + up256(R * I / 2);
    if (xsf_off + R * H / 16 > L.hq || hsf_off + R * I / 16 > L.out_acc) return MOE_ERR_INVALID_ARG;
    int* status = reinterpret_cast<int*>(b + L.status);
    int32_t* m_indptr = reinterpret_cast<int32_t*>(b + L.m_indptr);
    int32_t* perm = reinterpret_cast<int32_t*>(b + L.perm);
    int32_t* inv_perm = reinterpret_cast<int32_t*>(b + L.inv_perm);
    uint8_t* xq = reinterpret_cast<uint8_t*>(b + L.xq);
    uint8_t* xsf = reinterpret_cast<uint8_t*>(b + xsf_off);
    uint8_t* hq = reinterpret_cast<uint8_t*>(b + L.hq);
    uint8_t* hsf = reinterpret_cast<uint8_t*>(b + hsf_off);
    float* out_acc = reinterpret_cast<float*>(b + L.out_acc);
    if (cudaMemsetAsync(status, 0, sizeof(int) * kStatusInts, s) != cudaSuccess) return MOE_ERR_CUDA;
    RouteArgs ra{topk_ids, T, k, E, m_indptr, perm, inv_perm,
                 reinterpret_cast<int32_t*>(b + L.chunk_hist), status};
    stage_mark(0, s);
    int st = launch_route_permute(ra, s);
    if (st) return st;
    stage_mark(1, s);
    if (T > 0) {
        // x's scales are written row-major (coalesced per destination row) into the
        // intermediate's region, free until GEMM1, then made K-block-major; when that
        // region is too small (I < H/16) the scatter writes them K-block-major itself
        if (R * H / 16 <= L.out_acc - L.hq) {
            st = launch_nv_quant_scatter(x, T, H, k, a1_gscale, inv_perm, xq, hq,
                                         static_cast<int>(R), 0, out_acc, s);
            if (!st) st = launch_nv_sf_kblock_major(hq, xsf, static_cast<int>(R), H, s);
        } else {
            st = launch_nv_quant_scatter(x, T, H, k, a1_gscale, inv_perm, xq, xsf,
                                         static_cast<int>(R), 1, out_acc, s);
        }
        if (st) return st;
        stage_mark(2, s);
        const unsigned long long tmo = g_timeout_ns.load();
        NvGemmArgs g1{};
        g1.a = xq; g1.b = w13; g1.a_sf = xsf; g1.a_sf_mn = 1; g1.b_sf = w13_sf; g1.alpha = w13_alpha;
        g1.m_indptr = m_indptr; g1.R = static_cast<int>(R); g1.N = 2 * I; g1.K = H; g1.E = E;
        g1.gated = 1; g1.epi = NV_EPI_SWIGLU_NVQUANT; g1.hq = hq; g1.hsf = hsf;
        g1.h_gscale = a2_gscale;
        g1.status = status; g1.timeout_ns = tmo; g1.num_sms = d->sms;
        st = launch_nvfp4_gemm(g1, s);
        if (st) return st;
        stage_mark(3, s);
        NvGemmArgs g2{};
        g2.a = hq; g2.b = w2; g2.a_sf = hsf; g2.a_sf_mn = 1; g2.b_sf = w2_sf; g2.alpha = w2_alpha;
        g2.m_indptr = m_indptr; g2.R = static_cast<int>(R); g2.N = H; g2.K = I; g2.E = E;
        g2.gated = 0; g2.epi = NV_EPI_COMBINE; g2.perm = perm; g2.topk_w = topk_w; g2.topk = k;
        g2.out_acc = out_acc; g2.out_ld = H;
        g2.status = status; g2.timeout_ns = tmo; g2.num_sms = d->sms;
        st = launch_nvfp4_gemm(g2, s);
        if (st) return st;
        stage_mark(4, s);
        st = launch_f32_to_bf16(out_acc, out, static_cast<long long>(T) * H, d->sms, s);
        if (st) return st;
        stage_mark(5, s);
    }
    if (dbg_m_indptr &&
        cudaMemcpyAsync(dbg_m_indptr, m_indptr, sizeof(int32_t) * (E + 1), cudaMemcpyDeviceToDevice, s))
        return MOE_ERR_CUDA;
    if (R > 0) {
        if (dbg_perm &&
            cudaMemcpyAsync(dbg_perm, perm, sizeof(int32_t) * R, cudaMemcpyDeviceToDevice, s))
            return MOE_ERR_CUDA;
        if (dbg_hq && cudaMemcpyAsync(dbg_hq, hq, R * I / 2, cudaMemcpyDeviceToDevice, s))
            return MOE_ERR_CUDA;
        if (dbg_hsf && cudaMemcpyAsync(dbg_hsf, hsf, R * I / 16, cudaMemcpyDeviceToDevice, s))
            return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

int moe_nvfp4_fused(const void* x, const int32_t* topk_ids, const float* topk_w, const void* w13,
                    const uint8_t* w13_sf, const float* w13_alpha, const void* w2,
                    const uint8_t* w2_sf, const float* w2_alpha, float a1_gscale, float a2_gscale,
                    void* out, int T, int H, int I, int E, int k, void* ws, size_t ws_bytes,
                    moe_stream_t stream) {
    return nv_fused_impl(x, topk_ids, topk_w, w13, w13_sf, w13_alpha, w2, w2_sf, w2_alpha,
                         a1_gscale, a2_gscale, out, T, H, I, E, k, ws, ws_bytes, stream, nullptr,
                         nullptr, nullptr, nullptr);
}

int moe_nvfp4_fused_debug(const void* x, const int32_t* topk_ids, const float* topk_w,
                          const void* w13, const uint8_t* w13_sf, const float* w13_alpha,
                          const void* w2, const uint8_t* w2_sf, const float* w2_alpha,
                          float a1_gscale, float a2_gscale, void* out, int T, int H, int I, int E,
                          int k, void* ws, size_t ws_bytes, moe_stream_t stream, int32_t* m_indptr,
                          int32_t* perm, uint8_t* h_fp4, uint8_t* h_sf) {
    return nv_fused_impl(x, topk_ids, topk_w, w13, w13_sf, w13_alpha, w2, w2_sf, w2_alpha,
                         a1_gscale, a2_gscale, out, T, H, I, E, k, ws, ws_bytes, stream, m_indptr,
                         perm, h_fp4, h_sf);
}

int moe_fp8_fused(const void* x, const int32_t* topk_ids, const float* topk_w, const void* w13,
                  const float* w13_scale, const void* w2, const float* w2_scale, void* out, int T,
                  int H, int I, int E, int k, void* ws, size_t ws_bytes, moe_stream_t stream) {
    return fused_impl(x, topk_ids, topk_w, w13, w13_scale, w2, w2_scale, out, T, H, I, E, k, ws,
                      ws_bytes, stream, nullptr, nullptr, nullptr, nullptr);
}

int moe_fp8_fused_debug(const void* x, const int32_t* topk_ids, const float* topk_w, const void* w13,
                        const float* w13_scale, const void* w2, const float* w2_scale, void* out,
                        int T, int H, int I, int E, int k, void* ws, size_t ws_bytes,
                        moe_stream_t stream, int32_t* m_indptr, int32_t* perm, uint8_t* h_fp8,
                        float* h_scale) {
    return fused_impl(x, topk_ids, topk_w, w13, w13_scale, w2, w2_scale, out, T, H, I, E, k, ws,
                      ws_bytes, stream, m_indptr, perm, h_fp8, h_scale);
}

int fp8_groupwise_moe_gemm(const void* a, const void* b, const float* a_scale, const float* b_scale,
                           const int32_t* m_indptr, void* out, int R, int N, int K, int E,
                           int scale_major_mode, int sg_m, int sg_n, int sg_k, int is_gated,
                           int tile_m, int tile_n, moe_stream_t stream) {
    if (R < 0 || N <= 0 || K <= 0 || E < 1 || N % 128 || K % 128) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (scale_major_mode != 0 && scale_major_mode != 1) return MOE_ERR_INVALID_ARG;
    if (sg_m != 1 || sg_n != 128 || sg_k != 128) return MOE_ERR_UNSUPPORTED;
    // gated (fused SwiGLU) needs an even N: gate rows then up rows
    if (is_gated && (N % 2 || (N / 2) % 128)) return MOE_ERR_INVALID_ARG;
    if (!m_indptr || (R > 0 && (!a || !b || !a_scale || !b_scale || !out))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(b) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    const int want_tn = is_gated ? 128 : 256;
    if (tile_n != -1 && tile_n != want_tn) return MOE_ERR_NO_TILE_CONFIG;
    if (tile_m != -1 && tile_m != 16 && tile_m != 32 && tile_m != 64 && tile_m != 128)
        return MOE_ERR_NO_TILE_CONFIG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(d->lib_status, 0, sizeof(int) * kStatusInts, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (R == 0) return MOE_OK;
    int tm = tile_m;
    if (tm == -1) tm = choose_tile_m(R, N, K, E, is_gated, d->sms);
    if (tm < 128 && K > swap_max_k(tm)) {
        if (tile_m != -1) return MOE_ERR_NO_TILE_CONFIG;
        tm = fit_tile_to_k(tm, K);
    }
    GemmArgs g{};
    g.a = a; g.b = b; g.R = R; g.N = N; g.K = K; g.E = E;
    g.a_scale = a_scale;
    if (scale_major_mode == 0) { g.as_row = K / 128; g.as_kb = 1; }
    else { g.as_row = 1; g.as_kb = R; }
    g.b_scale = b_scale; g.m_indptr = m_indptr;
    g.epi = is_gated ? EPI_SWIGLU_BF16 : EPI_BF16;
    g.tile_m = tm;
    g.out_bf16 = out;
    g.status = d->lib_status;
    g.timeout_ns = g_timeout_ns.load();
    g.num_sms = d->sms;
    return launch_grouped_gemm(g, s);
}

int moe_tactic_tune_gemm(const void* a, const void* b, const float* a_scale, const float* b_scale,
                         const int32_t* m_indptr, void* out, int R, int N, int K, int E,
                         int scale_major_mode, int is_gated, int iters, moe_stream_t stream,
                         int* tile_m) {
    if (!tile_m || iters < 1 || R <= 0 || E < 1) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaEvent_t ev[2];
    if (cudaEventCreate(&ev[0]) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaEventCreate(&ev[1]) != cudaSuccess) {
        cudaEventDestroy(ev[0]);
        return MOE_ERR_CUDA;
    }
    int best = -1, st = MOE_OK;
    float best_ms = 0.0f;
    for (int tm : {16, 32, 64, 128}) {
        if (tm < 128 && K > swap_max_k(tm)) continue;
        auto run = [&]() {
            return fp8_groupwise_moe_gemm(a, b, a_scale, b_scale, m_indptr, out, R, N, K, E,
                                          scale_major_mode, 1, 128, 128, is_gated, tm, -1, stream);
        };
        if ((st = run()) != MOE_OK) break;  // warm-up
        if (cudaEventRecord(ev[0], s) != cudaSuccess) { st = MOE_ERR_CUDA; break; }
        for (int i = 0; i < iters && st == MOE_OK; ++i) st = run();
        if (st != MOE_OK) break;
        float ms = 0.0f;
        if (cudaEventRecord(ev[1], s) != cudaSuccess || cudaEventSynchronize(ev[1]) != cudaSuccess ||
            cudaEventElapsedTime(&ms, ev[0], ev[1]) != cudaSuccess) {
            st = MOE_ERR_CUDA;
            break;
        }
        if ((st = moe_get_device_status(nullptr, stream)) != MOE_OK) break;
        if (best < 0 || ms < best_ms) { best = tm; best_ms = ms; }
    }
    cudaEventDestroy(ev[0]);
    cudaEventDestroy(ev[1]);
    if (st != MOE_OK) return st;
    if (best < 0) return MOE_ERR_NO_TILE_CONFIG;
    tactic_store(TacticKey{N, K, E, is_gated ? 1 : 0, rows_bucket(R, E)}, best);
    *tile_m = best;
    return MOE_OK;
}

int moe_tactic_lookup(int R, int N, int K, int E, int is_gated, int* tile_m) {
    if (!tile_m || R < 0 || N <= 0 || K <= 0 || E < 1) return MOE_ERR_INVALID_ARG;
    return tactic_lookup(TacticKey{N, K, E, is_gated ? 1 : 0, rows_bucket(R, E)}, tile_m)
               ? MOE_OK
               : MOE_ERR_NO_TILE_CONFIG;
}

int moe_tactic_store(int R, int N, int K, int E, int is_gated, int tile_m) {
    if (R < 0 || N <= 0 || K <= 0 || E < 1) return MOE_ERR_INVALID_ARG;
    if (!valid_tile_m(tile_m) || (tile_m < 128 && K > swap_max_k(tile_m)))
        return MOE_ERR_NO_TILE_CONFIG;
    tactic_store(TacticKey{N, K, E, is_gated ? 1 : 0, rows_bucket(R, E)}, tile_m);
    return MOE_OK;
}

void moe_tactic_clear(void) {
    std::lock_guard<std::mutex> lk(g_tactic_mu);
    g_tactics.clear();
}

int moe_router_topk(const float* logits, int T, int E, int k, int32_t* topk_ids, float* topk_w,
                    moe_stream_t stream) {
    if (T < 0 || E < 1 || k < 1 || k > E || k > MOE_ROUTER_MAX_K) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (T > 0 && (!logits || !topk_ids || !topk_w)) return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    return launch_router_topk(logits, T, E, k, topk_ids, topk_w,
                              reinterpret_cast<cudaStream_t>(stream));
}

int moe_router_route(const float* logits, int T, int E, int k, int32_t* topk_ids, float* topk_w,
                     int32_t* m_indptr, int32_t* perm, int32_t* inv_perm, void* ws, size_t ws_bytes,
                     moe_stream_t stream) {
    if (T < 0 || E < 1 || k < 1 || k > E || k > MOE_ROUTER_MAX_K) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (!m_indptr || !ws || (T > 0 && (!logits || !topk_ids || !topk_w || !perm)))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < route_ws_bytes(T, k, E) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* base = static_cast<char*>(ws);
    int* status = reinterpret_cast<int*>(base);
    if (cudaMemsetAsync(status, 0, sizeof(int) * kStatusInts, s) != cudaSuccess) return MOE_ERR_CUDA;
    RouteArgs ra{topk_ids, T, k, E, m_indptr, perm, inv_perm,
                 reinterpret_cast<int32_t*>(base + up256(sizeof(int) * kStatusInts)), status};
    return launch_router_route(logits, ra, topk_w, s);
}

int mxfp8_moe_gemm(const void* a, const void* b, const uint8_t* a_sf, const uint8_t* b_sf,
                   const int32_t* m_indptr, void* out, int R, int N, int K, int E,
                   int a_sf_major, int is_gated, moe_stream_t stream) {
    if (R < 0 || N <= 0 || K <= 0 || E < 1 || N % 128 || K % 128) return MOE_ERR_INVALID_ARG;
    if (a_sf_major != 0 && a_sf_major != 1) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (is_gated && (N % 2 || (N / 2) % 128)) return MOE_ERR_INVALID_ARG;
    if (!m_indptr || (R > 0 && (!a || !b || !a_sf || !b_sf || !out))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(b) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(a_sf) & 3) || !aligned16(b_sf)) return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(d->lib_status, 0, sizeof(int) * kStatusInts, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (R == 0) return MOE_OK;
    MxGemmArgs g{};
    g.a = a; g.b = b; g.a_sf = a_sf; g.b_sf = b_sf; g.m_indptr = m_indptr;
    g.a_sf_mn = a_sf_major;
    g.R = R; g.N = N; g.K = K; g.E = E; g.gated = is_gated ? 1 : 0;
    g.epi = MX_EPI_BF16;
    g.out = out;
    g.status = d->lib_status;
    g.timeout_ns = g_timeout_ns.load();
    g.num_sms = d->sms;
    return launch_mx_gemm(g, s);
}

int mxfp8_tile_scales(const uint8_t* sf_rowmajor, uint8_t* sf_tiled, int rows, int K,
                      moe_stream_t stream) {
    if (rows < 0 || K <= 0 || K % 128 || rows % 128) return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!sf_rowmajor || !sf_tiled)) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(sf_rowmajor) | reinterpret_cast<uintptr_t>(sf_tiled)) & 3)
        return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    return launch_mx_tile_scales(sf_rowmajor, sf_tiled, rows, K, d->sms,
                                 reinterpret_cast<cudaStream_t>(stream));
}

int nvfp4_moe_gemm(const void* a, const void* b, const uint8_t* a_sf, const uint8_t* b_sf,
                   const float* alpha, const int32_t* m_indptr, void* out, int R, int N, int K,
                   int E, int a_sf_major, int is_gated, moe_stream_t stream) {
    if (R < 0 || N <= 0 || K <= 0 || E < 1 || N % 128 || K % 256) return MOE_ERR_INVALID_ARG;
    if (a_sf_major != 0 && a_sf_major != 1) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (is_gated && (N % 2 || (N / 2) % 128)) return MOE_ERR_INVALID_ARG;
    if (!m_indptr || (R > 0 && (!a || !b || !a_sf || !b_sf || !alpha || !out)))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(b) || !aligned16(out) || !aligned16(b_sf))
        return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(a_sf) | reinterpret_cast<uintptr_t>(alpha)) & 3)
        return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(d->lib_status, 0, sizeof(int) * kStatusInts, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (R == 0) return MOE_OK;
    NvGemmArgs g{};
    g.a = a; g.b = b; g.a_sf = a_sf; g.a_sf_mn = a_sf_major; g.b_sf = b_sf; g.alpha = alpha;
    g.m_indptr = m_indptr;
    g.R = R; g.N = N; g.K = K; g.E = E; g.gated = is_gated ? 1 : 0;
    g.out = out;
    g.status = d->lib_status;
    g.timeout_ns = g_timeout_ns.load();
    g.num_sms = d->sms;
    return launch_nvfp4_gemm(g, s);
}

int nvfp4_quantize(const void* x, float gscale, uint8_t* q, uint8_t* sf, int M, int K,
                   moe_stream_t stream) {
    if (M < 0 || K <= 0 || K % 128 || !(gscale > 0.0f)) return MOE_ERR_INVALID_ARG;
    if (M > 0 && (!x || !q || !sf)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(q) & 7)) return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    return launch_nv_quant_scatter(x, M, K, 1, gscale, nullptr, q, sf, M, 0, nullptr,
                                   reinterpret_cast<cudaStream_t>(stream));
}

int nvfp4_tile_scales(const uint8_t* sf_rowmajor, uint8_t* sf_tiled, int rows, int K,
                      moe_stream_t stream) {
    if (rows < 0 || K <= 0 || K % 64 || rows % 128) return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!sf_rowmajor || !sf_tiled)) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(sf_rowmajor) | reinterpret_cast<uintptr_t>(sf_tiled)) & 3)
        return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    // K/16 scales per row in groups of four: the MXFP8 tiling of a 2K-wide row
    // (2K/32 = K/16 scales, 2K/128 = K/64 groups)
    return launch_mx_tile_scales(sf_rowmajor, sf_tiled, rows, 2 * K, d->sms,
                                 reinterpret_cast<cudaStream_t>(stream));
}

int swiglu_mxfp8_quant(const void* in, void* out, uint8_t* scale, int M, int K, moe_stream_t stream) {
    if (M < 0 || K <= 0 || K % 32) return MOE_ERR_INVALID_ARG;
    if (M > 0 && (!in || !out || !scale)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(in) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // one launch per call: the kernel clears the status word itself
    if (M == 0 && cudaMemsetAsync(d->lib_status, 0, sizeof(int) * kStatusInts, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return launch_swiglu_mxfp8(in, out, scale, M, K, d->sms, d->lib_status, s);
}

// ---------------------------------------------------------------- expert parallelism
namespace {

// Workspace of moe_ep_plan: status word, owner rank per pair, chunk histograms.
struct EpPlanWs {
    size_t status, owner, chunk_hist, total;
};
EpPlanWs ep_plan_layout(int T, int k, int G) {
    const size_t R = static_cast<size_t>(T) * k;
    const size_t nchunks = (R + kRouteChunk - 1) / kRouteChunk;
    EpPlanWs w{};
    size_t o = 0;
    w.status = o;     o += up256(sizeof(int) * kStatusInts);
    w.owner = o;      o += up256(sizeof(int32_t) * R);
    w.chunk_hist = o; o += up256(sizeof(int32_t) * nchunks * G);
    w.total = o;
    return w;
}

// Workspace of moe_fp8_expert_rows, in carve order.
struct ExpertRowsWs {
    size_t status, m_indptr, chunk_hist, perm, inv_perm, xq, xs, hq, hs, total;
};
ExpertRowsWs expert_rows_layout(int n, int H, int I, int E) {
    const size_t N = static_cast<size_t>(n);
    const size_t nchunks = (N + kRouteChunk - 1) / kRouteChunk;
    ExpertRowsWs w{};
    size_t o = 0;
    w.status = o;     o += up256(sizeof(int) * kStatusInts);
    w.m_indptr = o;   o += up256(sizeof(int32_t) * (E + 1));
    w.chunk_hist = o; o += up256(sizeof(int32_t) * nchunks * E);
    w.perm = o;       o += up256(sizeof(int32_t) * N);
    w.inv_perm = o;   o += up256(sizeof(int32_t) * N);
    w.xq = o;         o += up256(N * H);
    w.xs = o;         o += up256(sizeof(float) * N * (H / 128));
    w.hq = o;         o += up256(N * I);
    w.hs = o;         o += up256(sizeof(float) * N * (I / 128));
    w.total = o;
    return w;
}

}  // namespace

size_t moe_ep_workspace_size(int T, int k, int G) {
    if (T < 0 || k < 1 || G < 1) return 0;
    return ep_plan_layout(T, k, G).total;
}

int moe_ep_plan(const int32_t* topk_ids, int T, int k, int E, int G, int32_t* send_indptr,
                int32_t* send_pair, int32_t* slot_of_pair, void* ws, size_t ws_bytes,
                moe_stream_t stream) {
    if (T < 0 || k < 1 || E < 1 || G < 1 || E % G || G > MOE_MAX_EXPERTS || E > MOE_MAX_EXPERTS)
        return MOE_ERR_INVALID_ARG;
    if (!send_indptr || !ws || (T > 0 && (!topk_ids || !send_pair || !slot_of_pair)))
        return MOE_ERR_INVALID_ARG;
    const EpPlanWs L = ep_plan_layout(T, k, G);
    if (ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    int* status = reinterpret_cast<int*>(b + L.status);
    int32_t* owner = reinterpret_cast<int32_t*>(b + L.owner);
    if (cudaMemsetAsync(status, 0, sizeof(int) * kStatusInts, s) != cudaSuccess) return MOE_ERR_CUDA;
    const long long R = static_cast<long long>(T) * k;
    int st = launch_ep_owner(topk_ids, R, E, E / G, owner, d->sms, s);
    if (st) return st;
    RouteArgs ra{owner, T, k, G, send_indptr, send_pair, slot_of_pair,
                 reinterpret_cast<int32_t*>(b + L.chunk_hist), status};
    return launch_route_permute(ra, s);
}

int moe_ep_pack(const void* x, const int32_t* topk_ids, const int32_t* slot_of_pair, int T, int H,
                int k, int E, int G, int S, uint8_t* xq_send, float* xs_send, int32_t* eid_send,
                moe_stream_t stream) {
    if (T < 0 || H <= 0 || H % 128 || k < 1 || E < 1 || G < 1 || E % G || S < 0)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !topk_ids || !slot_of_pair)) return MOE_ERR_INVALID_ARG;
    if (S > 0 && (!xq_send || !xs_send || !eid_send)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(xq_send) || (reinterpret_cast<uintptr_t>(xs_send) & 3))
        return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    return launch_ep_pack(x, topk_ids, T, H, k, S, slot_of_pair, E / G, xq_send, xs_send, eid_send,
                          reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_fp8_expert_rows_workspace_size(int n, int H, int I, int E) {
    if (n < 0 || H <= 0 || I <= 0 || E < 1) return 0;
    return expert_rows_layout(n, H, I, E).total;
}

int moe_fp8_expert_rows(const uint8_t* xq, const float* xs, const int32_t* eid, int n,
                        const void* w13, const float* w13_scale, const void* w2,
                        const float* w2_scale, float* y, int H, int I, int E, void* ws,
                        size_t ws_bytes, moe_stream_t stream) {
    if (n < 0 || H <= 0 || I <= 0 || H % 128 || I % 128 || E < 1) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (!ws) return MOE_ERR_INVALID_ARG;
    const ExpertRowsWs L = expert_rows_layout(n, H, I, E);
    if (ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    if (n > 0) {
        if (!xq || !xs || !eid || !w13 || !w13_scale || !w2 || !w2_scale || !y)
            return MOE_ERR_INVALID_ARG;
        if (!aligned16(xq) || !aligned16(w13) || !aligned16(w2) || !aligned16(y))
            return MOE_ERR_INVALID_ARG;
    }
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    int* status = reinterpret_cast<int*>(b + L.status);
    int32_t* m_indptr = reinterpret_cast<int32_t*>(b + L.m_indptr);
    int32_t* perm = reinterpret_cast<int32_t*>(b + L.perm);
    int32_t* inv_perm = reinterpret_cast<int32_t*>(b + L.inv_perm);
    uint8_t* hq = reinterpret_cast<uint8_t*>(b + L.hq);
    float* hs = reinterpret_cast<float*>(b + L.hs);
    if (cudaMemsetAsync(status, 0, sizeof(int) * kStatusInts, s) != cudaSuccess) return MOE_ERR_CUDA;
    // rows grouped by local expert (a stable sort of the row index)
    RouteArgs ra{eid, n, 1, E, m_indptr, perm, inv_perm,
                 reinterpret_cast<int32_t*>(b + L.chunk_hist), status};
    int st = launch_route_permute(ra, s);
    if (st || n == 0) return st;
    const unsigned long long tmo = g_timeout_ns.load();
    const int tm1 = fit_tile_to_k(choose_tile_m(n, 2 * I, H, E, 1, d->sms), H);
    const int tm2 = fit_tile_to_k(choose_tile_m(n, H, I, E, 0, d->sms), I);
    // grouped row r is received row perm[r]: swapped GEMM1 tiles read it (and
    // its row-major scales) there through the row map; 128-token tiles read a
    // grouped copy; GEMM2 writes the row back at perm[r]
    GemmArgs g1{};
    g1.b = w13; g1.R = n; g1.N = 2 * I; g1.K = H; g1.E = E; g1.b_scale = w13_scale;
    if (tm1 < 128) {
        g1.a = xq; g1.a_scale = xs; g1.as_row = H / 128; g1.as_kb = 1;
        g1.a_rowmap = perm; g1.a_rowdiv = 1; g1.a_rows = n;
    } else {
        uint8_t* xq_g = reinterpret_cast<uint8_t*>(b + L.xq);
        float* xs_g = reinterpret_cast<float*>(b + L.xs);
        st = launch_gather_rows(xq, xs, n, H, perm, n, m_indptr + E, xq_g, xs_g, s);
        if (st) return st;
        g1.a = xq_g; g1.a_scale = xs_g; g1.as_row = 1; g1.as_kb = n;
    }
    g1.m_indptr = m_indptr; g1.epi = EPI_SWIGLU_QUANT; g1.tile_m = tm1;
    g1.hq = hq; g1.hs = hs; g1.status = status; g1.timeout_ns = tmo; g1.num_sms = d->sms;
    st = launch_grouped_gemm(g1, s);
    if (st) return st;
    GemmArgs g2{};
    g2.a = hq; g2.b = w2; g2.R = n; g2.N = H; g2.K = I; g2.E = E;
    g2.a_scale = hs; g2.as_row = 1; g2.as_kb = n; g2.b_scale = w2_scale;
    g2.m_indptr = m_indptr; g2.epi = EPI_Y32; g2.tile_m = tm2;
    g2.y = y; g2.ldy = H; g2.rowmap = perm;
    g2.status = status; g2.timeout_ns = tmo; g2.num_sms = d->sms;
    return launch_grouped_gemm(g2, s);
}

int moe_combine(const float* y, const int32_t* row_of_pair, const float* topk_w, int T, int k, int H,
                void* out, moe_stream_t stream) {
    if (T < 0 || k < 1 || H <= 0 || H % 8) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!y || !topk_w || !out)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    const DevInfo* d = dev_info();
    if (int st = check_device(d)) return st;
    return launch_combine(y, row_of_pair, topk_w, T, k, H, out, reinterpret_cast<cudaStream_t>(stream));
}

int moe_get_device_status(const void* ws, moe_stream_t stream) {
    const DevInfo* d = dev_info();
    if (!d) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return MOE_ERR_CUDA;
    int h[kStatusInts] = {0, 0, 0, 0};
    const void* src = ws ? ws : d->lib_status;
    if (cudaMemcpy(h, src, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    return h[0];
}

}  // extern "C"
