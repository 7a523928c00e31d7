// api.cu -- the C ABI of libgqa.so (declared in include/gqa.h): argument
// checks, split planning, TMA tensor maps, the per-device workspace and the
// launches.  Everything here is host code except the device status word.
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>
#include <unordered_map>

#include "../../include/gqa.h"
#include "internal.h"
#include "mla.h"

namespace {

using namespace gqa;

__device__ int g_status_word;  // first error a kernel recorded (0 = none)
static_assert(kStatusTimeout == GQA_ERR_DEVICE_TIMEOUT, "device and host timeout codes differ");
static_assert(kStatusMisaligned == GQA_ERR_MISALIGNED, "device and host alignment codes differ");

constexpr unsigned long long kWaitBudgetNs = 1000000000ull;  // a bounded wait gives up after ~1 s
constexpr size_t kWorkspaceBudget = size_t(256) << 20;        // split partials of one call, at most

struct DeviceState {
    void *ws = nullptr;
    size_t ws_bytes = 0;
    int num_sms = 0;
    int *status = nullptr;
};

// Where workspaces come from: cudaMalloc / cudaFree, or the caller's pair (gqa_set_workspace_allocator).
struct WorkspaceAllocator {
    gqa_alloc_fn alloc = nullptr;
    gqa_free_fn free_fn = nullptr;
    void *ctx = nullptr;
};

std::mutex g_mu;
WorkspaceAllocator g_alloc;
std::unordered_map<int, DeviceState> g_devices;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
cudaEvent_t g_ev_before = nullptr, g_ev_after = nullptr;
thread_local int g_last_launches = 0;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gqa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA; }

// Per-device state (SM count, status-word address); caller holds g_mu.
gqa_status device_state(DeviceState **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
    DeviceState &st = g_devices[dev];
    if (st.num_sms == 0) {
        if (cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return GQA_ERR_CUDA;
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return GQA_ERR_CUDA;
        st.status = static_cast<int *>(p);
    }
    *out = &st;
    return GQA_OK;
}

// Hands a workspace block back to whoever allocated it; `dev` is current.  A caller's pool may reuse
// the block at once, so the device is synchronised first (cudaFree does the same implicitly).
void workspace_free(void *p, size_t bytes, int dev)
{
    if (!p) return;
    if (g_alloc.free_fn) {
        cudaDeviceSynchronize();
        g_alloc.free_fn(p, bytes, dev, g_alloc.ctx);
    } else {
        cudaFree(p);
    }
}

// Caller holds g_mu; the state's device is current.
gqa_status ensure_workspace(DeviceState *st, size_t bytes)
{
    if (bytes <= st->ws_bytes) return GQA_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
    workspace_free(st->ws, st->ws_bytes, dev);
    st->ws = nullptr;
    st->ws_bytes = 0;
    void *p = nullptr;
    if (g_alloc.alloc) {
        p = g_alloc.alloc(bytes, dev, g_alloc.ctx);
    } else if (cudaMalloc(&p, bytes) != cudaSuccess) {
        cudaGetLastError();
        p = nullptr;
    }
    if (!p) return GQA_ERR_OUT_OF_MEMORY;
    if (reinterpret_cast<uintptr_t>(p) & 255u) {   // the partials and the piece list assume 256-byte alignment
        workspace_free(p, bytes, dev);
        return GQA_ERR_MISALIGNED;
    }
    st->ws = p;
    st->ws_bytes = bytes;
    return GQA_OK;
}

// Hands back every device's workspace (caller holds g_mu); the current device is restored.
void release_workspaces()
{
    if (g_devices.empty()) return;
    int cur = 0;
    cudaGetDevice(&cur);
    for (auto &kv : g_devices) {
        if (kv.second.ws) {
            cudaSetDevice(kv.first);
            workspace_free(kv.second.ws, kv.second.ws_bytes, kv.first);
            kv.second.ws = nullptr;
            kv.second.ws_bytes = 0;
        }
    }
    cudaSetDevice(cur);
}

gqa_status get_encoder()
{
    if (g_encode) return GQA_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return GQA_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return GQA_OK;
}

// 4-D bf16 map over a [n3][n2][n1][n0] row-major tensor, box {64, 1, rows, 1},
// 128-byte swizzle: one box is `rows` rows of one 64-column half of a head.
gqa_status encode_4d(CUtensorMap *tm, const void *base, uint64_t n0, uint64_t n1, uint64_t n2, uint64_t n3,
                     uint32_t box_rows)
{
    cuuint64_t dims[4] = {n0, n1, n2, n3};
    cuuint64_t strides[3] = {n0 * 2, n0 * n1 * 2, n0 * n1 * n2 * 2};
    cuuint32_t box[4] = {64, 1, box_rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_CUDA;
}

// 4-D map over E4M3 codes [n3][n2][n1][128] (one byte each), box {128, 1, rows, 1}, 128-byte swizzle:
// one box is `rows` whole rows of one head.
gqa_status encode_4d_codes(CUtensorMap *tm, const void *base, uint64_t n1, uint64_t n2, uint64_t n3,
                           uint32_t box_rows)
{
    const uint64_t n0 = kHeadDim;
    cuuint64_t dims[4] = {n0, n1, n2, n3};
    cuuint64_t strides[3] = {n0, n0 * n1, n0 * n1 * n2};
    cuuint32_t box[4] = {(cuuint32_t)n0, 1, box_rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_CUDA;
}

gqa_status check_decode_args(const void *q, const void *k, const void *v, const int32_t *seqlens, int B, int Hq,
                             int Hkv, int d, int Tmax, const void *out)
{
    if (!q || !k || !v || !seqlens || !out) return GQA_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Tmax <= 0) return GQA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return GQA_ERR_INVALID_ARG;
    if (d != kHeadDim) return GQA_ERR_UNSUPPORTED;
    if (B > 65535 || Hq > 65535) return GQA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return GQA_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(seqlens) & 3u) return GQA_ERR_MISALIGNED;
    return GQA_OK;
}

gqa_status run_decode(const void *q, const void *k, const void *v, const int32_t *seqlens, int B, int Hq, int Hkv,
                      int Tmax, float scale, void *out, cudaStream_t stream, int *launches,
                      const Fp8Scales *fp8 = nullptr);

}  // namespace

namespace gqa {

int *device_status_word()
{
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState *st = nullptr;
    return device_state(&st) == GQA_OK ? st->status : nullptr;
}

void set_last_launch_count(int n) { g_last_launches = n; }

static size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

DecodePlan decode_plan_host(int B, int Hq, int Hkv, int Tmax, int num_sms, size_t ws_budget, bool fp8)
{
    const int g = Hq / Hkv;
    DecodeShape sh = decode_shape(g);
    if (fp8) {
        // the FP8 kernel is the tensor-core one for every group size it takes (g <= 32)
        sh.tensor_cores = true;
        sh.tile = 128;
        sh.heads_per_cta = g;
        sh.nhb = 1;
        sh.ctas_per_sm = 1;
    }
    DecodePlan p{};
    p.tile = sh.tile;
    p.hb = sh.heads_per_cta;
    p.nhb = sh.nhb;
    p.tensor_cores = sh.tensor_cores;
    const long long tiles = (Tmax + sh.tile - 1) / sh.tile;
    if (sh.tensor_cores) {
        // the device cuts histories from the real lengths (decode_plan_kernel); the host only bounds
        // the pieces per sequence (at most 64, fewer when their partials would not fit the budget)
        // and sizes the workspace for that bound
        const size_t per_piece = (size_t)B * Hq * (kHeadDim + 2) * 4 + (size_t)B * 16;
        long long cap = 64;
        if (cap > tiles) cap = tiles;
        const long long fit = per_piece ? (long long)(ws_budget / per_piece) : cap;
        if (fit < cap) cap = fit < 1 ? 1 : fit;
        if (tiles <= kStaticPlanTiles) {
            p.static_plan = true;
            p.nsplit = 1;
            p.chunk = (int)(tiles * sh.tile);
            p.ws_bytes = 0;
            return p;
        }
        const long long cmin = (tiles + cap - 1) / cap;
        p.nsplit = (int)((tiles + cmin - 1) / cmin);
        p.chunk = (int)(cmin * sh.tile);
        size_t off = 0;
        p.off_hdr = off;
        off += 256;
        p.off_nsb = off;
        off += round256((size_t)B * 4);   // pieces per sequence
        p.off_items = off;
        off += round256((size_t)B * p.nsplit * 16);
        p.off_po = off;
        off += round256((size_t)B * Hq * p.nsplit * kHeadDim * 4);
        p.off_pml = off;
        off += round256((size_t)B * Hq * p.nsplit * 2 * 4);
        p.ws_bytes = off;
        return p;
    }
    const long long base = (long long)B * Hkv * p.nhb;
    const long long slots = (long long)num_sms * sh.ctas_per_sm;
    // cost in units of "one stage per resident CTA": waves x (tiles per split + start-up),
    // plus the partials' round trip and one extra launch when the history is split
    double best = 1e300;
    int best_s = 1;
    const long long smax = tiles < 4096 ? tiles : 4096;
    for (long long s = 1; s <= smax; ++s) {
        const long long ct = (tiles + s - 1) / s;
        const long long se = (tiles + ct - 1) / ct;
        if (se != s) continue;
        // split partials must fit the workspace budget; one piece per sequence needs none
        if (se > 1 && (double)B * Hq * se * (kHeadDim + 2) * 4.0 > (double)ws_budget) continue;
        const long long waves = (base * se + slots - 1) / slots;
        // each CTA also pays a fixed start-up (barriers, query rows, pipeline fill): about one tile
        double cost = (double)waves * ((double)ct + 1.0);
        if (se > 1) {
            const double part_bytes = 2.0 * B * Hq * se * (kHeadDim + 2) * 4.0;
            cost += part_bytes / (double)(sh.tile * 512) / (double)slots + 2.0 * kDecodeTile / sh.tile;
        }
        if (cost < best - 1e-9) {
            best = cost;
            best_s = (int)se;
        }
    }
    p.chunk = (int)(((tiles + best_s - 1) / best_s) * sh.tile);
    p.nsplit = (Tmax + p.chunk - 1) / p.chunk;
    p.off_po = 0;
    p.off_pml = (size_t)B * Hq * p.nsplit * kHeadDim * 4;
    p.ws_bytes = p.nsplit > 1 ? (size_t)B * Hq * p.nsplit * (kHeadDim + 2) * sizeof(float) : 0;
    return p;
}

int decode_enqueue(const void *q, const void *k, const void *v, const int32_t *seqlens, int B, int Hq, int Hkv,
                   int Tmax, float scale, void *out, void *ws, const DecodePlan &p, int num_sms, int *status,
                   cudaStream_t stream, int *launches, cudaEvent_t ev_before, cudaEvent_t ev_after,
                   const Fp8Scales *fp8)
{
    gqa_status s;
    if ((s = get_encoder()) != GQA_OK) return s;
    if ((long long)Hkv * p.nhb > 65535) return GQA_ERR_UNSUPPORTED;
    if (p.ws_bytes > 0 && !ws) return GQA_ERR_INVALID_ARG;
    if (fp8 && (!p.tensor_cores || p.tile != 128 || Hq / Hkv > 32)) return GQA_ERR_UNSUPPORTED;
    CUtensorMap tmK, tmV, tmQ;
    if (fp8) {
        if ((s = encode_4d_codes(&tmK, k, Hkv, Tmax, B, 128)) != GQA_OK) return s;
        if ((s = encode_4d_codes(&tmV, v, Hkv, Tmax, B, 128)) != GQA_OK) return s;
    } else {
        if ((s = encode_4d(&tmK, k, kHeadDim, Hkv, Tmax, B, p.tile)) != GQA_OK) return s;
        if ((s = encode_4d(&tmV, v, kHeadDim, Hkv, Tmax, B, p.tile)) != GQA_OK) return s;
    }

    uint8_t *w = static_cast<uint8_t *>(ws);
    DecodeArgs a{};
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.seqlens = seqlens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.part_o = w ? reinterpret_cast<float *>(w + p.off_po) : nullptr;
    a.part_ml = w ? reinterpret_cast<float *>(w + p.off_pml) : nullptr;
    a.status = status;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Tmax = Tmax;
    a.group = Hq / Hkv;
    a.chunk = p.chunk;
    a.nsplit = p.nsplit;
    a.nhb = p.nhb;
    a.qscale = scale * 1.4426950408889634f;  // log2(e): the softmax runs in base 2
    if (fp8) {
        a.qk_factor = a.qscale * fp8->k_scale;
        a.o_factor = fp8->v_scale * (1.0f / 128.0f);
    }
    a.wait_budget_ns = kWaitBudgetNs;
    a.num_ctas = num_sms;
    // groups of 9-16 are planned in two rounds of long pieces with their remainders cut in two, larger
    // groups in one round with remainders cut in four (sweeps over rounds and tail pieces: +2-3 % at
    // g = 16; at g = 32, +1-1.5 % bf16 and +3 % FP8 over two rounds)
    a.tail_split = a.group > 16 ? 4 : (a.group > 8 ? 2 : 1);
    int n = 0;
    if (p.tensor_cores) {
        // the group's query rows as a 3-D map (d, heads, batch): one box = N rows of one 64-column half
        const int N = a.group <= 16 ? 16 : 32;
        cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)Hq, (cuuint64_t)B};
        cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)kHeadDim * Hq * 2};
        cuuint32_t box[3] = {64, (cuuint32_t)N, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return GQA_ERR_CUDA;
    }
    if (p.tensor_cores && p.static_plan) {
        // one launch: whole histories as units, nothing to plan or combine
        a.static_plan = 1;
        if (ev_before) cudaEventRecord(ev_before, stream);
        if ((s = cuda_status(launch_decode_tc(tmK, tmV, tmQ, a, stream, fp8 != nullptr))) != GQA_OK) return s;
        if (ev_after) cudaEventRecord(ev_after, stream);
        ++n;
    } else if (p.tensor_cores) {
        a.plan_hdr = reinterpret_cast<int *>(w + p.off_hdr);
        a.nsplit_b = reinterpret_cast<int *>(w + p.off_nsb);
        a.items = reinterpret_cast<int4 *>(w + p.off_items);
        if ((s = cuda_status(launch_decode_plan(a, stream))) != GQA_OK) return s;
        ++n;
        if (ev_before) cudaEventRecord(ev_before, stream);
        if ((s = cuda_status(launch_decode_tc(tmK, tmV, tmQ, a, stream, fp8 != nullptr))) != GQA_OK) return s;
        if (ev_after) cudaEventRecord(ev_after, stream);
        ++n;
        if ((s = cuda_status(launch_decode_combine(a, stream, true))) != GQA_OK) return s;
        ++n;
    } else {
        if (ev_before) cudaEventRecord(ev_before, stream);
        if ((s = cuda_status(launch_decode_split(tmK, tmV, a, stream))) != GQA_OK) return s;
        if (ev_after) cudaEventRecord(ev_after, stream);
        ++n;
        if (p.nsplit > 1) {
            if ((s = cuda_status(launch_decode_combine(a, stream))) != GQA_OK) return s;
            ++n;
        }
    }
    *launches += n;
    return GQA_OK;
}

}  // namespace gqa

namespace {

gqa_status run_decode(const void *q, const void *k, const void *v, const int32_t *seqlens, int B, int Hq, int Hkv,
                      int Tmax, float scale, void *out, cudaStream_t stream, int *launches,
                      const Fp8Scales *fp8)
{
    DeviceState *st = nullptr;
    gqa_status s = device_state(&st);
    if (s != GQA_OK) return s;
    const DecodePlan p = decode_plan_host(B, Hq, Hkv, Tmax, st->num_sms, kWorkspaceBudget, fp8 != nullptr);
    if (p.ws_bytes > 0 && (s = ensure_workspace(st, p.ws_bytes)) != GQA_OK) return s;
    return static_cast<gqa_status>(decode_enqueue(q, k, v, seqlens, B, Hq, Hkv, Tmax, scale, out, st->ws, p,
                                                  st->num_sms, st->status, stream, launches, g_ev_before,
                                                  g_ev_after, fp8));
}

}  // namespace

extern "C" {

gqa_status gqa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens, int B, int Hq,
                      int Hkv, int d, int Tmax, float scale, void *out, void *stream)
{
    g_last_launches = 0;
    gqa_status s = check_decode_args(q, k_cache, v_cache, seqlens, B, Hq, Hkv, d, Tmax, out);
    if (s != GQA_OK) return s;
    std::lock_guard<std::mutex> lk(g_mu);
    return run_decode(q, k_cache, v_cache, seqlens, B, Hq, Hkv, Tmax, scale, out,
                      static_cast<cudaStream_t>(stream), &g_last_launches);
}

gqa_status gqa_decode_fp8(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens, int B,
                          int Hq, int Hkv, int d, int Tmax, float scale, float k_scale, float v_scale, void *out,
                          void *stream)
{
    g_last_launches = 0;
    gqa_status s = check_decode_args(q, k_cache, v_cache, seqlens, B, Hq, Hkv, d, Tmax, out);
    if (s != GQA_OK) return s;
    if (!std::isfinite(scale) || !std::isfinite(k_scale) || !std::isfinite(v_scale)) return GQA_ERR_INVALID_ARG;
    if (Hq / Hkv > 32) return GQA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    const Fp8Scales sc{k_scale, v_scale};
    return run_decode(q, k_cache, v_cache, seqlens, B, Hq, Hkv, Tmax, scale, out,
                      static_cast<cudaStream_t>(stream), &g_last_launches, &sc);
}

size_t gqa_decode_expanded_bytes(int B, int Tmax, int Hq, int d)
{
    if (B <= 0 || Tmax <= 0 || Hq <= 0 || d <= 0) return 0;
    return (size_t)B * (size_t)Tmax * (size_t)Hq * (size_t)d * 2u;
}

gqa_status gqa_decode_expanded(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
                               int B, int Hq, int Hkv, int d, int Tmax, float scale, void *out, void *k_rep,
                               void *v_rep, void *stream)
{
    g_last_launches = 0;
    gqa_status s = check_decode_args(q, k_cache, v_cache, seqlens, B, Hq, Hkv, d, Tmax, out);
    if (s != GQA_OK) return s;
    if (!k_rep || !v_rep) return GQA_ERR_INVALID_ARG;
    if (!aligned16(k_rep) || !aligned16(v_rep)) return GQA_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lk(g_mu);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((s = cuda_status(launch_repeat_kv(k_cache, v_cache, seqlens, k_rep, v_rep, B, Tmax, Hq, Hkv, st))) != GQA_OK)
        return s;
    g_last_launches = 1;
    return run_decode(q, k_rep, v_rep, seqlens, B, Hq, Hq, Tmax, scale, out, st, &g_last_launches);
}

// Host checks shared by both MLA decode entry points.
static gqa_status check_mla_args(const void *q, const void *kv_cache, const int32_t *seqlens, int B, int Hq, int d_c,
                                 int d_r, int Tmax, const void *out)
{
    if (!q || !kv_cache || !seqlens || !out) return GQA_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || d_c <= 0 || d_r < 0 || Tmax <= 0) return GQA_ERR_INVALID_ARG;
    if (d_c != kMlaLatent || d_r != kMlaRope) return GQA_ERR_UNSUPPORTED;
    if (B > 65535 || Hq > 65535) return GQA_ERR_UNSUPPORTED;   // grid dimensions
    if (!aligned16(q) || !aligned16(kv_cache) || !aligned16(out)) return GQA_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(seqlens) & 3u) return GQA_ERR_MISALIGNED;
    return GQA_OK;
}

// 3-D bf16 map over a [n2][n1][n0] row-major tensor, box {64, rows, 1}, 128-byte swizzle.
static gqa_status encode_3d(CUtensorMap *tm, const void *base, uint64_t n0, uint64_t n1, uint64_t n2,
                            uint32_t box_rows)
{
    cuuint64_t dims[3] = {n0, n1, n2};
    cuuint64_t strides[2] = {n0 * 2, n0 * n1 * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_CUDA;
}

// A [n2][rows][576] bf16 tensor viewed as (64 columns, rows, 9 column chunks, n2): the chunk index is
// outside the row index, so one box {64, box_rows, chunks, 1} lands in shared memory as `chunks`
// consecutive tiles of box_rows x 64 columns (128-byte swizzle), the layout the MMA descriptors read.
static gqa_status encode_chunk_view(CUtensorMap *tm, const void *base, uint64_t rows, uint64_t n2, uint32_t box_rows,
                                    uint32_t chunks)
{
    cuuint64_t dims[4] = {64, rows, (cuuint64_t)(kMlaRow / 64), n2};
    cuuint64_t strides[3] = {(cuuint64_t)kMlaRow * 2, 128, rows * kMlaRow * 2};
    cuuint32_t box[4] = {64, box_rows, chunks, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_CUDA;
}

gqa_status gqa_mla_decode(const void *q, const void *kv_cache, const int32_t *seqlens, int B, int Hq, int d_c,
                          int d_r, int Tmax, float scale, void *out, void *stream)
{
    g_last_launches = 0;
    gqa_status s = check_mla_args(q, kv_cache, seqlens, B, Hq, d_c, d_r, Tmax, out);
    if (s != GQA_OK) return s;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState *st = nullptr;
    if ((s = device_state(&st)) != GQA_OK) return s;
    if ((s = get_encoder()) != GQA_OK) return s;
    const MlaTcPlan p = mla_tc_plan_host(B, Hq, Tmax, kWorkspaceBudget);
    if ((s = ensure_workspace(st, p.ws_bytes)) != GQA_OK) return s;
    CUtensorMap tmKV2, tmKV1, tmQ;
    if ((s = encode_chunk_view(&tmKV2, kv_cache, Tmax, B, 128, 2)) != GQA_OK) return s;
    if ((s = encode_3d(&tmKV1, kv_cache, kMlaRow, Tmax, B, 128)) != GQA_OK) return s;
    if ((s = encode_chunk_view(&tmQ, q, Hq, B, 64, kMlaRow / 64)) != GQA_OK) return s;
    int n = 0;
    const cudaError_t e = launch_mla_decode_tc(tmKV2, tmKV1, tmQ, q, seqlens, B, Hq, Tmax, scale, out, st->ws, p,
                                               st->num_sms, st->status, kWaitBudgetNs,
                                               static_cast<cudaStream_t>(stream), &n, g_ev_before, g_ev_after);
    g_last_launches = n;
    return cuda_status(e);
}

gqa_status gqa_mla_decode_cudacore(const void *q, const void *kv_cache, const int32_t *seqlens, int B, int Hq,
                                   int d_c, int d_r, int Tmax, float scale, void *out, void *stream)
{
    g_last_launches = 0;
    gqa_status s = check_mla_args(q, kv_cache, seqlens, B, Hq, d_c, d_r, Tmax, out);
    if (s != GQA_OK) return s;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState *st = nullptr;
    if ((s = device_state(&st)) != GQA_OK) return s;
    const MlaPlan p = mla_plan_host(B, Hq, Tmax, st->num_sms);
    if (p.ws_bytes > 0 && (s = ensure_workspace(st, p.ws_bytes)) != GQA_OK) return s;
    MlaArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.kv = static_cast<const __nv_bfloat16 *>(kv_cache);
    a.seqlens = seqlens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.part_o = p.nsplit > 1 ? static_cast<float *>(st->ws) : nullptr;
    a.part_ml = p.nsplit > 1 ? a.part_o + (size_t)B * Hq * p.nsplit * kMlaLatent : nullptr;
    a.B = B;
    a.Hq = Hq;
    a.Tmax = Tmax;
    a.nsplit = p.nsplit;
    a.chunk = p.chunk;
    a.qscale = scale * 1.4426950408889634f;
    int n = 0;
    const cudaError_t e = launch_mla_decode(a, static_cast<cudaStream_t>(stream), &n, g_ev_before, g_ev_after);
    g_last_launches = n;
    return cuda_status(e);
}

gqa_status gqa_tp_shard(int Hq, int Hkv, int tp, int rank, int *q_first, int *q_count, int *kv_first,
                        int *kv_count)
{
    if (!q_first || !q_count || !kv_first || !kv_count) return GQA_ERR_INVALID_ARG;
    if (Hq <= 0 || Hkv <= 0 || tp <= 0 || rank < 0 || rank >= tp || Hq % Hkv != 0) return GQA_ERR_INVALID_ARG;
    // ranks own consecutive, equal runs of query heads
    if (Hq % tp != 0) return GQA_ERR_UNSUPPORTED;
    const int g = Hq / Hkv, nq = Hq / tp;
    int kf = 0, kc = 0;
    if (Hkv >= tp) {
        // partition: each rank owns Hkv / tp whole KV heads, and with them exactly its query heads' groups
        if (Hkv % tp != 0) return GQA_ERR_UNSUPPORTED;
        kc = Hkv / tp;
        kf = rank * kc;
    } else {
        // replication: the rank's query heads lie in one group; it keeps a copy of that group's KV head
        if (tp % Hkv != 0) return GQA_ERR_UNSUPPORTED;
        kc = 1;
        kf = (rank * nq) / g;
    }
    *q_first = rank * nq;
    *q_count = nq;
    *kv_first = kf;
    *kv_count = kc;
    return GQA_OK;
}

gqa_status gqa_decode_plan(int B, int Hq, int Hkv, int d, int Tmax, int num_sms, int *chunk, int *nsplit,
                           size_t *workspace_bytes)
{
    if (!chunk || !nsplit || !workspace_bytes) return GQA_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Tmax <= 0 || num_sms <= 0) return GQA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return GQA_ERR_INVALID_ARG;
    if (d != kHeadDim) return GQA_ERR_UNSUPPORTED;
    const DecodePlan p = decode_plan_host(B, Hq, Hkv, Tmax, num_sms, kWorkspaceBudget);
    *chunk = p.chunk;
    *nsplit = p.nsplit;
    *workspace_bytes = p.ws_bytes;
    return GQA_OK;
}

}  // extern "C"

namespace {

gqa_status check_prefill_args(const void *q, const void *k, const void *v, int B, int S, int Hq, int Hkv, int d,
                              const void *out)
{
    if (!q || !k || !v || !out) return GQA_ERR_INVALID_ARG;
    if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return GQA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return GQA_ERR_INVALID_ARG;
    if (d != kHeadDim) return GQA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return GQA_ERR_MISALIGNED;
    if (B > 65535 || S > (1 << 30)) return GQA_ERR_UNSUPPORTED;
    return GQA_OK;
}

gqa_status run_prefill(const void *q, const void *k, const void *v, int B, int S, int Hq, int Hkv, int d, void *out,
                       float *lse, void *stream)
{
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState *st = nullptr;
    gqa_status s = device_state(&st);
    if (s != GQA_OK) return s;
    if ((s = get_encoder()) != GQA_OK) return s;
    CUtensorMap tmQ, tmK, tmV;
    if ((s = encode_4d(&tmQ, q, kHeadDim, Hq, S, B, 128)) != GQA_OK) return s;
    if ((s = encode_4d(&tmK, k, kHeadDim, Hkv, S, B, 128)) != GQA_OK) return s;
    if ((s = encode_4d(&tmV, v, kHeadDim, Hkv, S, B, 128)) != GQA_OK) return s;
    PrefillArgs a;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.status = st->status;
    a.B = B;
    a.S = S;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.group = Hq / Hkv;
    a.qscale = 1.4426950408889634f / std::sqrt((float)d);   // log2(e) / sqrt(d): base-2 softmax
    a.wait_budget_ns = kWaitBudgetNs;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (g_ev_before) cudaEventRecord(g_ev_before, cs);
    if ((s = cuda_status(launch_prefill(tmQ, tmK, tmV, a, cs))) != GQA_OK) return s;
    if (g_ev_after) cudaEventRecord(g_ev_after, cs);
    g_last_launches = 1;
    return GQA_OK;
}

}  // namespace

extern "C" {

gqa_status gqa_prefill_causal(const void *q, const void *k, const void *v, int B, int S, int Hq, int Hkv, int d,
                              void *out, void *stream)
{
    g_last_launches = 0;
    gqa_status s = check_prefill_args(q, k, v, B, S, Hq, Hkv, d, out);
    if (s != GQA_OK) return s;
    return run_prefill(q, k, v, B, S, Hq, Hkv, d, out, nullptr, stream);
}

gqa_status gqa_prefill_causal_fwd(const void *q, const void *k, const void *v, int B, int S, int Hq, int Hkv,
                                  int d, void *out, float *lse, void *stream)
{
    g_last_launches = 0;
    gqa_status s = check_prefill_args(q, k, v, B, S, Hq, Hkv, d, out);
    if (s != GQA_OK) return s;
    if (!lse) return GQA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(lse) & 3u) return GQA_ERR_MISALIGNED;
    return run_prefill(q, k, v, B, S, Hq, Hkv, d, out, lse, stream);
}

gqa_status gqa_prefill_causal_bwd(const void *q, const void *k, const void *v, const void *out, const float *lse,
                                  const void *dout, int B, int S, int Hq, int Hkv, int d, void *dq, void *dk,
                                  void *dv, void *stream)
{
    g_last_launches = 0;
    gqa_status s = check_prefill_args(q, k, v, B, S, Hq, Hkv, d, out);
    if (s != GQA_OK) return s;
    if (!lse || !dout || !dq || !dk || !dv) return GQA_ERR_INVALID_ARG;
    if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return GQA_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(lse) & 3u) return GQA_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState *st = nullptr;
    if ((s = device_state(&st)) != GQA_OK) return s;
    if ((s = get_encoder()) != GQA_OK) return s;
    const size_t dbytes = (size_t)B * Hq * S * sizeof(float);
    if ((s = ensure_workspace(st, dbytes)) != GQA_OK) return s;
    CUtensorMap tmQ, tmK, tmV, tmDO;
    if ((s = encode_4d(&tmQ, q, kHeadDim, Hq, S, B, 128)) != GQA_OK) return s;
    if ((s = encode_4d(&tmK, k, kHeadDim, Hkv, S, B, 128)) != GQA_OK) return s;
    if ((s = encode_4d(&tmV, v, kHeadDim, Hkv, S, B, 128)) != GQA_OK) return s;
    if ((s = encode_4d(&tmDO, dout, kHeadDim, Hq, S, B, 128)) != GQA_OK) return s;
    BackwardArgs a;
    a.out = static_cast<const __nv_bfloat16 *>(out);
    a.dout = static_cast<const __nv_bfloat16 *>(dout);
    a.lse = lse;
    a.dsum = static_cast<float *>(st->ws);
    a.dq = static_cast<__nv_bfloat16 *>(dq);
    a.dk = static_cast<__nv_bfloat16 *>(dk);
    a.dv = static_cast<__nv_bfloat16 *>(dv);
    a.status = st->status;
    a.B = B;
    a.S = S;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.group = Hq / Hkv;
    a.scale = 1.0f / std::sqrt((float)d);
    a.qscale = 1.4426950408889634f * a.scale;
    a.wait_budget_ns = kWaitBudgetNs;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    int n = 0;
    if (g_ev_before) cudaEventRecord(g_ev_before, cs);
    s = cuda_status(launch_prefill_backward(tmQ, tmK, tmV, tmDO, a, cs, &n));
    if (g_ev_after) cudaEventRecord(g_ev_after, cs);
    g_last_launches = n;
    return s;
}

gqa_status gqa_get_last_device_status(void *stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return GQA_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof(int)) != cudaSuccess) return GQA_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int)) != cudaSuccess) return GQA_ERR_CUDA;
    return static_cast<gqa_status>(v);
}

gqa_status gqa_selftest_wait_timeout(int timeout_us, void *stream)
{
    g_last_launches = 0;
    if (timeout_us <= 0 || timeout_us > 10000000) return GQA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState *st = nullptr;
    gqa_status s = device_state(&st);
    if (s != GQA_OK) return s;
    s = cuda_status(launch_wait_timeout_selftest(st->status, (unsigned long long)timeout_us * 1000ull,
                                                 static_cast<cudaStream_t>(stream)));
    if (s == GQA_OK) g_last_launches = 1;
    return s;
}

gqa_status gqa_set_profile_events(void *before, void *after)
{
    std::lock_guard<std::mutex> lk(g_mu);
    if ((before == nullptr) != (after == nullptr)) return GQA_ERR_INVALID_ARG;
    g_ev_before = static_cast<cudaEvent_t>(before);
    g_ev_after = static_cast<cudaEvent_t>(after);
    return GQA_OK;
}

int gqa_last_launch_count(void) { return g_last_launches; }

void gqa_release(void)
{
    std::lock_guard<std::mutex> lk(g_mu);
    release_workspaces();
    g_devices.clear();
}

gqa_status gqa_set_workspace_allocator(gqa_alloc_fn alloc, gqa_free_fn free_fn, void *ctx)
{
    if ((alloc == nullptr) != (free_fn == nullptr)) return GQA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    release_workspaces();   // each block goes back to the allocator that made it
    g_alloc.alloc = alloc;
    g_alloc.free_fn = free_fn;
    g_alloc.ctx = alloc ? ctx : nullptr;
    return GQA_OK;
}

const char *gqa_status_string(gqa_status s)
{
    switch (s) {
    case GQA_OK: return "ok";
    case GQA_ERR_INVALID_ARG: return "invalid argument";
    case GQA_ERR_UNSUPPORTED: return "unsupported shape";
    case GQA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case GQA_ERR_OUT_OF_MEMORY: return "workspace allocation failed";
    case GQA_ERR_CUDA: return "CUDA error";
    case GQA_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
    }
    return "unknown status";
}

const char *gqa_version(void) { return "gqa-b200 0.1"; }

}  // extern "C"
