// decode_tc.cu -- GQA decode with the dot products on the tcgen05 tensor cores,
// scheduled from the actual sequence lengths.
//
// Per (sequence b, KV head) the group's g query heads are the N dimension of
// two small matrix products per 128-token tile, with the tokens as the
// 128-row M dimension:
//
//   S^T [128 tokens x N] = K_tile [128 x d] . Q_g^T           (A = K, K-major; B = Q, K-major)
//   O^T [d x N]         += V_tile^T [d x 128] . P^T [128 x N]  (A = V, MN-major; B = P^T, MN-major)
//
// N is g rounded up to 16 or 32.  Each K/V tile is fetched from HBM once by TMA
// and serves every head of the group ("Kernels do not need to copy the KV
// heads", anrans.github.io attention-variants: the group's query heads become
// extra rows against one shared KV head).  The softmax weights enter the
// second product as two bf16 terms (hi + lo), so the result carries them to
// about 2^-17 relative, like an fp32 weight.
//
// Scheduling.  The host cannot see the lengths (they live on the device), so
// decode_plan_kernel reads them and cuts every history into pieces of C tiles,
// C chosen from the total work so that there are about eight rounds of pieces
// (two for groups above 16), and lists the pieces longest first.  decode_persistent_kernel then runs one
// CTA per SM; each CTA claims (piece, KV head) units from an atomic counter
// and keeps its TMA / MMA / softmax pipeline running across units.  A unit
// that covers its whole history writes the output; otherwise it writes a
// partial result (o, m, l) that decode_combine_kernel merges.  The three
// kernels are chained with programmatic dependent launch, so each one's
// launch and prologue overlap the previous one.
//
// The softmax runs on one 128-thread warpgroup per 16 heads, one token per
// thread (TMEM lane = token for S^T, lane = d for O^T).  The running maximum
// of each head only moves when some score exceeds it by more than 8 (log2
// units); in the common case a tile costs one warp vote and one group barrier.
//
// Warps: 0..4*nwg-1 softmax + epilogue (nwg = N/16), then (FP8 cache) the
// converter warpgroup, the TMA producer (it also claims units and loads the
// group's query rows), the TMEM allocator + S^T issuer, and the PV issuer.  The
// two products are issued by different threads so that S^T runs up to four
// tiles ahead instead of queueing behind the previous tile's PV product.
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace gqa {

namespace {

constexpr int kD = kHeadDim;
constexpr int kTok = 128;                 // tokens per tile (the M of S^T)
constexpr int kTile = kTok * kD * 2;      // 32 KB: one K or V tile
constexpr int kHalf = kTile / 2;          // one 64-column half
constexpr int kWG = 128;                  // threads of one softmax warpgroup (one token each)
constexpr int kQD = 4;                    // depth of the unit queue in shared memory
constexpr float kMoveThreshold = 8.0f;
constexpr int kPlanMaxC = 4096;           // remainder sizes sorted by a shared-memory histogram up to this

// barrier slots: each name owns a contiguous range (sizes checked against the configuration below)
enum : int { K_FULL = 0, V_FULL = 3, KV_EMPTY = 6, S_FULL = 9, S_FREE = 13, P_FULL = 17, P_FREE = 21, O_FULL = 25,
             O_FREE = 27, Q_FULL = 29, Q_EMPTY = 31, I_FULL = 33, I_EMPTY = 37, DRAIN = 41, DRAIN_PV = 42, GRP = 43,
             // FP8 only: code ring (R_EMPTY: the stage's PV product is done), converted V (in the stage),
             // the query's E4M3 terms, the unit slot's score factors (the softmax releases the slot after
             // reading them), and the stage's key codes read by the S^T products
             R_FULL = 47, R_EMPTY = 53, VC_FULL = 59, QC_FULL = 65, QF_FULL = 67, K_READ = 71,
             kBarSlots = 77 };
constexpr int kBarSlotsFor(bool f8) { return f8 ? kBarSlots : R_FULL; }
template <class C, bool F8>
constexpr bool barrier_ranges_fit()
{
    return (F8 ? C::stages <= 6 : C::stages <= 3) && C::sbufs <= 4 && C::pbufs <= 4 && C::nwg <= 4 && kQD <= 4;
}

// F8 = false: bf16 cache; the K and V tiles go from TMA straight to the tensor cores.
// F8 = true: FP8 (E4M3) cache.  TMA brings the raw code tiles (16 KB each) into a ring.  S^T is an
// E4M3 product (kind::f8f6f4) straight from the key codes: the query enters it as two E4M3 terms of
// q 2^e per head (t0 = e4m3(v), t1 = e4m3(v - t0), which carry a bf16 element exactly down to 2^-10
// of the head's largest |q| and within 2^-17 of it below), stacked as 2N rows of B, and the softmax adds
// the two products.  One
// converter warpgroup widens the values exactly to f16 (every E4M3 value is an f16 value) into a
// 128-byte-swizzled tile that takes the place of the stage's two code tiles, once S^T has read the
// keys.  P enters the second product as one f16 term of 128 p (so that small weights stay normal;
// relative rounding 2^-11 per weight, against the bf16 path's hi + lo pair), an f16 MMA.
// HW: heads one softmax warpgroup handles (4, 8 or 16), NWG: softmax warpgroups.  Groups of up to 4
// or 8 heads only compute their own columns of the N = 16 wide products; more warpgroups with fewer
// heads each shorten the softmax's per-tile chain.
template <int N, bool F8, int HW, int NWG>
struct TcCfg {
    static_assert(NWG * HW <= N && (NWG == 1 || HW % 8 == 0), "softmax heads within the product");
    static constexpr int nwg = NWG;                           // softmax warpgroups
    static constexpr int nb = NWG * HW <= 8 ? 1 : NWG * HW / 8;   // 8-head blocks of P^T / O^T that carry heads
    static constexpr int conv_warps = F8 ? 4 : 0;             // FP8: the converter warpgroup
    // + TMA warp + S^T issuer warp + PV issuer warp.  FP8 with 32 heads: the last three warps are padded
    // to a warpgroup and the registers are redistributed (setmaxnreg).  Two softmax warpgroups: 512
    // threads launch with 128 registers each, the softmax warpgroups then take 176, the converter 104
    // and the last warpgroup 56; four: 768 threads launch with 80, the softmax takes 88, the converter
    // 72 and the last warpgroup 40 (the sum never exceeds the launch's share, so every increase is covered
    // by the decreases).  Interleaved A/B at g = 32: with the keys multiplied as codes the converter only
    // widens the values, and 88/72 (no spills) is 2.7 % faster than 80/104 and 96/56.
    static constexpr bool regsplit = F8 && N == 32;
    static constexpr int threads = regsplit ? kWG * (nwg + 2) : kWG * nwg + 32 * conv_warps + 96;
    static constexpr int reg_launch = nwg == 4 ? 80 : 128;
    static constexpr int reg_soft = nwg == 4 ? 88 : 176;
    static constexpr int reg_conv = nwg == 4 ? 72 : 104;
    static constexpr int reg_last = nwg == 4 ? 40 : 56;
    static_assert(!regsplit || (nwg == 2 || nwg == 4), "register split for two or four softmax warpgroups");
    static_assert(!regsplit || kWG * (nwg * reg_soft + reg_conv + reg_last) <= threads * reg_launch,
                  "register split within the launch's share");
    static constexpr int sbufs = 4;                            // S^T buffers: QK^T runs up to four tiles ahead
    static constexpr int pbufs = (F8 || N == 16) ? 2 : 1;      // P^T buffers (2: the softmax runs a tile ahead)
    // P as one 16-bit term (FP8: f16 of 128 p, relative rounding 2^-11 on each weight) or as bf16 hi + lo
    // terms (bf16: 2^-8 on its own would be as coarse as the output's rounding)
    static constexpr int p_terms = F8 ? 1 : 2;
    static constexpr int stages = F8 ? (N == 32 ? 5 : 6) : 3;
    // K then V (FP8: two 16 KB code tiles, then the f16 V tile in their place)
    static constexpr int stage_bytes = F8 ? kTile : 2 * kTile;
    static constexpr int q_off = stages * stage_bytes;        // Q[2 buffers]: [2 halves][N rows][128 B], swizzled
    static constexpr int q_half = N * 128;
    static constexpr int q_bytes = 2 * q_half;
    static constexpr int p_off = q_off + 2 * q_bytes;         // P^T[pbufs]: hi blocks, then lo blocks,
    static constexpr int p_half = nb * 2048;                  //   each [16 token groups][8 tokens][8 heads] 16-bit
    static constexpr int red_off = p_off + pbufs * 2 * p_half; // [2][4][N] floats: tile maxima per warp
    static constexpr int lsum_off = red_off + 2 * 4 * N * 4;  // [2 O buffers][4][N] floats: l partials per warp
    static constexpr int mst_off = lsum_off + 2 * 4 * N * 4;  // [2 O buffers][N] floats: the unit's final maxima
    static constexpr int qfac_off = mst_off + 2 * N * 4;      // FP8: [kQD unit slots][N] score factors per head
    static constexpr int vote_off = qfac_off + (F8 ? kQD * N * 4 : 0);   // [nwg][2][4] ints
    static constexpr int queue_off = vote_off + nwg * 32;     // kQD units of 8 ints
    static constexpr int bar_off = queue_off + kQD * 32;
    static constexpr int nbars = kBarSlotsFor(F8);
    static constexpr int tmem_off = bar_off + nbars * 8;
    static constexpr int err_off = tmem_off + 8;
    static constexpr int bytes = err_off + 8;
    // FP8: K[2] (64 columns each: 128 f16 keys per token, packed in pairs) first, then as below.
    // S[sbufs] (N columns each) and O[2] (2N columns each: the hi and lo products side by side, the lo
    // columns 8 * nb after the hi ones; FP8 reads only the hi columns)
    // FP8: each S buffer holds the products with the query's two E4M3 terms side by side (2N columns)
    static constexpr uint32_t s_cols = F8 ? 2 * N : N;
    static constexpr uint32_t s_base = 0;
    static constexpr uint32_t o_base = s_base + sbufs * s_cols;
    static constexpr uint32_t tmem_used = o_base + 4 * N;
    static constexpr uint32_t tmem_cols = tmem_used <= 128 ? 128 : (tmem_used <= 256 ? 256 : 512);
    static_assert(bytes <= 227 * 1024, "shared memory budget");
};


__device__ __forceinline__ void record_status(int *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ bool wait_or_fail(uint64_t *bar, uint32_t parity, const DecodeArgs &a, volatile int *err)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*err) return false;
        if (global_timer_ns() - t0 > a.wait_budget_ns) {
            *err = 1;
            record_status(a.status, kStatusTimeout);
            return false;
        }
    }
    return true;
}

// Barrier among one warpgroup's 128 threads on an mbarrier, so that it gives up (bounded) like every
// other wait instead of blocking forever when another role has failed.  `uses` counts earlier syncs.
__device__ __forceinline__ bool group_sync(uint64_t *grp, int &uses, const DecodeArgs &a, volatile int *err)
{
    mbar_arrive(grp);
    const bool r = wait_or_fail(grp, uses & 1, a, err);
    ++uses;
    return r;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ int plan_tokens(const DecodeArgs &a, int b)
{
    const int T = __ldg(a.seqlens + b);
    return T < 0 ? 0 : (T > a.Tmax ? a.Tmax : T);
}

// Exclusive scan over the warp; *total receives the sum of all lanes' values.
__device__ __forceinline__ int warp_exclusive_scan(int v, int &total)
{
    const int lane = threadIdx.x & 31;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    total = __shfl_sync(0xffffffffu, x, 31);
    return x - v;
}

// Cuts every history into pieces of C tiles and lists them longest first:
// plan_hdr = {claim counter (reset to 0), pieces, C}; nsplit_b[b] = pieces of sequence b;
// items[i] = {b, piece index | pieces of b << 16, first token, end token}.  Full pieces come first, in
// sequence order, then the shorter last pieces in decreasing length (a counting sort).
// One warp: its time is latency (one read of the lengths and a few dependent steps), which a warp
// takes with shuffles where a larger block would need barriers.  The lengths are read once, eight
// coalesced loads in flight per lane, into shared memory; lane l then owns the contiguous sequences
// [l * per, (l + 1) * per).
constexpr int kPlanLenCache = 4096;   // lengths kept in shared memory (any further ones are re-read)

__global__ void __launch_bounds__(32) decode_plan_kernel(const DecodeArgs a, int slots)
{
    __shared__ int hist[kPlanMaxC];          // tail pieces per size class, then each class's next slot
    __shared__ int s_len[kPlanLenCache];     // clamped lengths of the first kPlanLenCache sequences

    // launched as a programmatic dependent of whatever ran before on the stream (the previous call's
    // combine, say, which still reads nsplit_b): wait for it before touching anything, so that only the
    // launch overlaps it
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the persistent kernel may start its prologue now; it reads this plan only after griddepcontrol.wait
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int lane = threadIdx.x;
    const int ncache = min(a.B, kPlanLenCache);
    for (int i0 = 0; i0 < ncache; i0 += 8 * 32) {
        int v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * 32 + lane;
            v[u] = i < ncache ? __ldg(a.seqlens + i) : 0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * 32 + lane;
            if (i < ncache) s_len[i] = v[u] < 0 ? 0 : (v[u] > a.Tmax ? a.Tmax : v[u]);
        }
    }
    __syncwarp();
    auto tokens = [&](int b) { return b < kPlanLenCache ? s_len[b] : plan_tokens(a, b); };
    const int per = (a.B + 31) / 32;
    const int b0 = min(a.B, lane * per), b1 = min(a.B, b0 + per);
    long long tot = 0;
    int mx = 0;
    for (int b = b0; b < b1; ++b) {
        const int tl = (tokens(b) + kTok - 1) / kTok;
        tot += tl;
        mx = max(mx, tl);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tot += __shfl_xor_sync(0xffffffffu, tot, o);
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    // rounds of (piece, KV head) units per persistent CTA: eight for groups up to 8, two up to 16 and one
    // above, whose units of more heads carry a larger fixed cost each (measured on the benchmark shapes);
    // never more than nsplit pieces
    const long long rounds = a.plan_rounds > 0 ? a.plan_rounds : (a.group > 16 ? 1 : (a.group > 8 ? 2 : 8));
    long long Cl = (tot * a.Hkv + rounds * slots - 1) / (rounds * slots);
    const long long cmin = (mx + a.nsplit - 1) / a.nsplit;
    if (Cl < cmin) Cl = cmin;
    if (Cl > mx) Cl = mx;
    if (Cl < 1) Cl = 1;
    const int C = (int)Cl;
    // remainder sizes sort by a shared histogram up to kPlanMaxC; past that they keep no order and
    // hist[0] counts and then places them
    const bool sort_rem = C <= kPlanMaxC;
    const int nclass = sort_rem ? C : 1;
    for (int i = lane; i < nclass; i += 32) hist[i] = 0;
    __syncwarp();
    // A history's remainder (tl % C tiles) is cut into up to tail_split pieces of nearly equal size
    // (never more than nsplit pieces in all): the shortest units are claimed last, so that the CTAs
    // finish together even when some of them stream their tiles more slowly than others.
    const int tsplit = a.tail_split > 1 ? a.tail_split : 1;
    auto tail_pieces = [&](int full, int rem) -> int {
        if (rem <= 0) return 0;
        int k = tsplit < rem ? tsplit : rem;
        if (k > a.nsplit - full) k = a.nsplit - full;
        return k > 1 ? k : 1;
    };
    int nfull = 0;
    bool empty = false;
    for (int b = b0; b < b1; ++b) {
        const int tl = (tokens(b) + kTok - 1) / kTok;
        const int full = tl / C, rem = tl % C;
        const int k = tail_pieces(full, rem);
        a.nsplit_b[b] = full + k;
        nfull += full;
        empty |= tl == 0;
        if (sort_rem) {
            for (int j = 0; j < k; ++j) {
                const int size = rem / k + (j < rem % k ? 1 : 0);
                atomicAdd(&hist[C - 1 - size], 1);   // reversed: longest first
            }
        } else if (k > 0) {
            atomicAdd(&hist[0], k);
        }
    }
    if (__any_sync(0xffffffffu, empty)) {
        // no cached token: no unit will touch such a sequence, its output rows are zero
        const int orow = a.out_row > 0 ? a.out_row : kD;
        for (int b = 0; b < a.B; ++b) {
            if (tokens(b) > 0) continue;
            uint4 *o = reinterpret_cast<uint4 *>(a.out + (size_t)b * a.Hq * orow);
            for (int i = lane; i < a.Hq * orow / 8; i += 32) o[i] = make_uint4(0, 0, 0, 0);
        }
    }
    __syncwarp();
    int F;
    int f0 = warp_exclusive_scan(nfull, F);   // first slot of this lane's full pieces
    // hist[C-1-r] becomes the first slot (after the full pieces) of the tail pieces of r tiles
    {
        const int cper = (nclass + 31) / 32;
        const int c0 = min(nclass, lane * cper), c1 = min(nclass, c0 + cper);
        int run = 0;
        for (int c = c0; c < c1; ++c) run += hist[c];
        int ntail;
        int base = F + warp_exclusive_scan(run, ntail);
        for (int c = c0; c < c1; ++c) {
            const int n = hist[c];
            hist[c] = base;
            base += n;
        }
        if (lane == 0) {
            a.plan_hdr[0] = 0;   // claim counter
            a.plan_hdr[1] = F + ntail;
            a.plan_hdr[2] = C;
        }
    }
    __syncwarp();
    for (int b = b0; b < b1; ++b) {
        const int T = tokens(b);
        const int tl = (T + kTok - 1) / kTok;
        const int full = tl / C, rem = tl % C;
        const int k = tail_pieces(full, rem);
        const int np_b = full + k;
        for (int s = 0; s < full; ++s)
            a.items[f0 + s] = make_int4(b, s | (np_b << 16), s * C * kTok, min((s + 1) * C * kTok, T));
        f0 += full;
        int start = full * C;   // first tile of the next tail piece
        for (int j = 0; j < k; ++j) {
            const int size = rem / k + (j < rem % k ? 1 : 0);
            const int pos = atomicAdd(&hist[sort_rem ? C - 1 - size : 0], 1);
            a.items[pos] = make_int4(b, (full + j) | (np_b << 16), start * kTok, min((start + size) * kTok, T));
            start += size;
        }
    }
}

// Two E4M3 codes (low byte first) -> f16x2, exact.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t w, uint32_t &lo, uint32_t &hi)
{
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}


// 32 lanes x 32 bits, NC (4, 8 or 16) consecutive columns per thread.
template <int NC>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t (&r)[NC])
{
    if constexpr (NC == 16) {
        tmem_ld16(taddr, r);
    } else if constexpr (NC == 8) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                       "=r"(r[7])
                     : "r"(taddr));
    } else {
        static_assert(NC == 4, "4, 8 or 16 columns");
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                     : "r"(taddr));
    }
}

template <int NC>
__device__ __forceinline__ void tmem_stn(uint32_t taddr, const uint32_t (&r)[NC])
{
    if constexpr (NC == 16) {
        tmem_st16(taddr, r);
    } else if constexpr (NC == 8) {
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                     "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                     : "memory");
    } else {
        static_assert(NC == 4, "4, 8 or 16 columns");
        asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]),
                     "r"(r[1]), "r"(r[2]), "r"(r[3])
                     : "memory");
    }
}

// The warp's register share becomes R (from L at launch): setmaxnreg.inc waits for the registers that
// other warps' setmaxnreg.dec release.
template <int R, int L>
__device__ __forceinline__ void set_max_regs()
{
    static_assert(R % 8 == 0 && R >= 24 && R <= 256, "setmaxnreg takes multiples of 8 in [24, 256]");
    if constexpr (R > L) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R) : "memory");
    else if constexpr (R < L) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R) : "memory");
}

// ---------------------------------------------------------------------------------------------
template <int N, bool F8, int HW, int NWG>
__global__ void __launch_bounds__(TcCfg<N, F8, HW, NWG>::threads, 1)
decode_persistent_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmQ, const DecodeArgs a)
{
    using C = TcCfg<N, F8, HW, NWG>;
    static_assert(barrier_ranges_fit<C, F8>(), "a barrier range is too small for this configuration");
    // the 128-byte swizzle needs 1024-byte aligned tiles; the whole budget is used, so there is no room
    // to realign: a misaligned window is reported and the CTA does nothing
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) record_status(a.status, kStatusMisaligned);
        return;
    }

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = a.group;

    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + C::bar_off);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::tmem_off);
    volatile int *err = reinterpret_cast<volatile int *>(smem + C::err_off);
    float *red = reinterpret_cast<float *>(smem + C::red_off);
    float *lsum = reinterpret_cast<float *>(smem + C::lsum_off);
    float *mst = reinterpret_cast<float *>(smem + C::mst_off);
    float *qfac = reinterpret_cast<float *>(smem + C::qfac_off);
    volatile int *vote = reinterpret_cast<volatile int *>(smem + C::vote_off);
    volatile int *queue = reinterpret_cast<volatile int *>(smem + C::queue_off);
    uint8_t *ps = smem + C::p_off;

    const int conv_warp0 = 4 * C::nwg;
    const int producer_warp = conv_warp0 + C::conv_warps, mma_warp = producer_warp + 1, pv_warp = mma_warp + 1;
    constexpr int unit_readers = 2 + kWG * C::nwg + 32 * C::conv_warps;   // 2 MMA issuers + softmax + converter
    if (threadIdx.x == 0) {
        if constexpr (F8) {
            for (int s = 0; s < C::stages; ++s) {
                mbar_init(&bar[R_FULL + s], 1);
                mbar_init(&bar[R_EMPTY + s], 1);
                mbar_init(&bar[VC_FULL + s], kWG);
                mbar_init(&bar[K_READ + s], 1);
            }
            for (int s = 0; s < 2; ++s) {
                mbar_init(&bar[QC_FULL + s], kWG);
            }
            for (int s = 0; s < kQD; ++s) mbar_init(&bar[QF_FULL + s], kWG);
        } else {
            for (int s = 0; s < C::stages; ++s) {
                mbar_init(&bar[K_FULL + s], 1);
                mbar_init(&bar[V_FULL + s], 1);
                mbar_init(&bar[KV_EMPTY + s], 1);
            }
        }
        for (int s = 0; s < C::sbufs; ++s) {
            mbar_init(&bar[S_FULL + s], 1);
            mbar_init(&bar[S_FREE + s], kWG * C::nwg);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[O_FULL + s], 1);
            mbar_init(&bar[O_FREE + s], kWG * C::nwg);
            mbar_init(&bar[Q_FULL + s], 1);
            mbar_init(&bar[Q_EMPTY + s], 1);
        }
        for (int s = 0; s < C::pbufs; ++s) {
            mbar_init(&bar[P_FULL + s], kWG * C::nwg);
            mbar_init(&bar[P_FREE + s], 1);
        }
        for (int s = 0; s < kQD; ++s) {
            mbar_init(&bar[I_FULL + s], 1);
            mbar_init(&bar[I_EMPTY + s], unit_readers);
        }
        mbar_init(&bar[DRAIN], 1);
        mbar_init(&bar[DRAIN_PV], 1);
        for (int w = 0; w < C::nwg; ++w) mbar_init(&bar[GRP + w], kWG);
        *err = 0;
        fence_barrier_init();
    }
    if (warp == mma_warp) {
        tmem_alloc(tmem_slot, C::tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // everything below may read what decode_plan_kernel wrote; the combine kernel may be scheduled
    // now (it waits for this grid to finish before it reads anything)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS0 = tmem + C::s_base;   // S buffer i at tS0 + i * s_cols
    // O buffer i at tO0 + 2N i: V^T P_hi^T, then (8 nb columns later) V^T P_lo^T
    const uint32_t tO0 = tmem + C::o_base;

    // Register split (FP8, 32 heads): each warpgroup sets its share first thing in its own branch, the
    // same instruction for all four of its warps (the shares are checked against the launch's in TcCfg).
    if (warp >= producer_warp) {
        // the last warpgroup: producer, S^T issuer, PV issuer (and, with the split, one idle warp)
        if constexpr (C::regsplit) set_max_regs<C::reg_last, C::reg_launch>();
        if (warp == producer_warp) {
            // ---------------- claims units, loads the group's query rows and streams the K/V tiles
            if (lane == 0) {
                tma_prefetch_desc(&tmK);
                tma_prefetch_desc(&tmV);
                tma_prefetch_desc(&tmQ);
                // static schedule (no planner): unit u = (sequence u / Hkv, KV head u % Hkv), the whole
                // history as one piece, units dealt round-robin over the CTAs
                const bool stat = a.static_plan != 0;
                const int units = stat ? a.B * a.Hkv : a.plan_hdr[1] * a.Hkv;
                int tcount = 0, icount = 0, issued_tiles = 0, claim = 0;
                while (true) {
                    int u = stat ? blockIdx.x + (claim++) * gridDim.x : atomicAdd(&a.plan_hdr[0], 1);
                    int4 it = make_int4(0, 0, 0, 0);
                    if (stat) {
                        // an empty history has no unit: its output rows are zero
                        for (; u < units; u = blockIdx.x + (claim++) * gridDim.x) {
                            const int bb = u / a.Hkv;
                            int T = a.seqlens[bb];
                            T = T < 0 ? 0 : (T > a.Tmax ? a.Tmax : T);
                            if (T > 0) {
                                it = make_int4(bb, 1 << 16, 0, T);   // piece 0 of 1
                                break;
                            }
                            uint4 *o = reinterpret_cast<uint4 *>(a.out + ((size_t)bb * a.Hq + (u % a.Hkv) * g) * kD);
                            for (int i = 0; i < g * kD / 8; ++i) o[i] = make_uint4(0, 0, 0, 0);
                        }
                    }
                    const int slot = icount % kQD;
                    if (icount >= kQD && !wait_or_fail(&bar[I_EMPTY + slot], ((icount / kQD) - 1) & 1, a, err)) break;
                    volatile int *q = queue + slot * 8;
                    if (u >= units) {
                        q[4] = -1;                         // no more work
                        mbar_arrive(&bar[I_FULL + slot]);
                        break;
                    }
                    if (!stat) it = a.items[u / a.Hkv];
                    const int kvh = u % a.Hkv;
                    q[0] = it.x;
                    q[1] = kvh;
                    q[2] = it.y;
                    q[3] = it.z;
                    q[4] = it.w;
                    mbar_arrive(&bar[I_FULL + slot]);
                    const int qb = icount & 1;
                    if (icount >= 2 && !wait_or_fail(&bar[Q_EMPTY + qb], ((icount >> 1) - 1) & 1, a, err)) break;
                    uint8_t *qs = smem + C::q_off + qb * C::q_bytes;
                    mbar_arrive_expect_tx(&bar[Q_FULL + qb], C::q_bytes);
                    tma_load_3d(qs, &tmQ, &bar[Q_FULL + qb], 0, kvh * g, it.x);
                    tma_load_3d(qs + C::q_half, &tmQ, &bar[Q_FULL + qb], 64, kvh * g, it.x);
                    const int ntl = (it.w - it.z + kTok - 1) / kTok;
                    bool ok = true;
                    for (int jj = 0; jj < ntl; ++jj, ++tcount) {
                        const int s = tcount % C::stages;
                        const int t0 = it.z + jj * kTok;
                        uint8_t *ks = smem + s * C::stage_bytes;
                        if constexpr (F8) {
                            if (tcount >= C::stages &&
                                !wait_or_fail(&bar[R_EMPTY + s], ((tcount / C::stages) - 1) & 1, a, err)) {
                                ok = false;
                                break;
                            }
                            // one box = 128 tokens x 128 one-byte codes of a head
                            mbar_arrive_expect_tx(&bar[R_FULL + s], kTile);
                            tma_load_4d(ks, &tmK, &bar[R_FULL + s], 0, kvh, t0, it.x);
                            tma_load_4d(ks + kHalf, &tmV, &bar[R_FULL + s], 0, kvh, t0, it.x);
                        } else {
                            if (tcount >= C::stages &&
                                !wait_or_fail(&bar[KV_EMPTY + s], ((tcount / C::stages) - 1) & 1, a, err)) {
                                ok = false;
                                break;
                            }
                            mbar_arrive_expect_tx(&bar[K_FULL + s], kTile);
                            tma_load_4d(ks, &tmK, &bar[K_FULL + s], 0, kvh, t0, it.x);
                            tma_load_4d(ks + kHalf, &tmK, &bar[K_FULL + s], 64, kvh, t0, it.x);
                            mbar_arrive_expect_tx(&bar[V_FULL + s], kTile);
                            tma_load_4d(ks + kTile, &tmV, &bar[V_FULL + s], 0, kvh, t0, it.x);
                            tma_load_4d(ks + kTile + kHalf, &tmV, &bar[V_FULL + s], 64, kvh, t0, it.x);
                        }
                        issued_tiles = tcount + 1;
                    }
                    ++icount;
                    if (!ok) break;
                }
                // leave no copy in flight
                for (int t = issued_tiles - 1; t >= 0 && t >= issued_tiles - C::stages; --t) {
                    const uint32_t ph = (t / C::stages) & 1;
                    if constexpr (F8) {
                        mbar_wait(&bar[R_FULL + t % C::stages], ph, a.wait_budget_ns);
                    } else {
                        mbar_wait(&bar[K_FULL + t % C::stages], ph, a.wait_budget_ns);
                        mbar_wait(&bar[V_FULL + t % C::stages], ph, a.wait_budget_ns);
                    }
                }
                for (int i = icount - 1; i >= 0 && i >= icount - 2; --i)
                    mbar_wait(&bar[Q_FULL + (i & 1)], (i >> 1) & 1, a.wait_budget_ns);
            }
        } else if (warp == mma_warp) {
            // ---------------- S^T issuer: S^T = K (K-major) . Q^T (K-major), as soon as the keys and a free
            // S buffer allow (up to four tiles ahead of the softmax)
            if (lane == 0) {
                const uint32_t idesc_s = F8 ? umma_idesc_f16(kTok, 2 * N, 0, 0) : umma_idesc_bf16(kTok, N, 0, 0);
                int tcount = 0, icount = 0;
                bool ok = true;
                while (ok) {
                    const int slot = icount % kQD;
                    if (!wait_or_fail(&bar[I_FULL + slot], (icount / kQD) & 1, a, err)) break;
                    volatile int *q = queue + slot * 8;
                    const int t_begin = q[3], t_end = q[4];
                    mbar_arrive(&bar[I_EMPTY + slot]);
                    if (t_end < 0) break;
                    const int ntl = (t_end - t_begin + kTok - 1) / kTok;
                    const int qb = icount & 1;
                    if (!wait_or_fail(&bar[(F8 ? QC_FULL : Q_FULL) + qb], (icount >> 1) & 1, a, err)) break;
                    const uint32_t q_addr = smem_u32(smem + C::q_off + qb * C::q_bytes);
                    for (int jj = 0; jj < ntl; ++jj) {
                        const int T = tcount + jj;
                        const int s = T % C::stages, sb = T % C::sbufs;
                        if (!wait_or_fail(&bar[(F8 ? R_FULL : K_FULL) + s], (T / C::stages) & 1, a, err)) {
                            ok = false;
                            break;
                        }
                        if (T >= C::sbufs &&
                            !wait_or_fail(&bar[S_FREE + sb], ((T / C::sbufs) - 1) & 1, a, err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d_tmem = tS0 + sb * C::s_cols;
                        if constexpr (F8) {
                            // A = the stage's key codes as TMA left them ([128 tokens][128 codes], 128-byte
                            // swizzle), B = the query's two E4M3 terms as 2N rows (term 0, then term 1): the
                            // keys cross shared memory once, 32 codes of K per product
                            const uint32_t k_addr = smem_u32(smem + s * C::stage_bytes);
    #pragma unroll
                            for (int ks = 0; ks < kD / 32; ++ks)
                                umma_ss_e4m3(d_tmem, umma_smem_desc(k_addr + ks * 32, 16, 1024, 2),
                                             umma_smem_desc(q_addr + ks * 32, 16, 1024, 2), idesc_s, ks > 0 ? 1u : 0u);
                            umma_commit(&bar[S_FULL + sb]);
                            umma_commit(&bar[K_READ + s]);   // the key codes may now be overwritten
                        } else {
                            const uint32_t k_addr = smem_u32(smem + s * C::stage_bytes);
    #pragma unroll
                            for (int ks = 0; ks < kD / 16; ++ks) {
                                const uint32_t ka = k_addr + (ks >> 2) * kHalf + (ks & 3) * 32;
                                const uint32_t qa = q_addr + (ks >> 2) * C::q_half + (ks & 3) * 32;
                                umma_ss(d_tmem, umma_smem_desc(ka, 16, 1024, 2), umma_smem_desc(qa, 16, 1024, 2),
                                        idesc_s, ks > 0 ? 1u : 0u);
                            }
                            umma_commit(&bar[S_FULL + sb]);
                        }
                    }
                    if (!ok) break;
                    umma_commit(&bar[Q_EMPTY + qb]);   // the unit's query rows are no longer read
                    tcount += ntl;
                    ++icount;
                }
                umma_commit(&bar[DRAIN]);
                mbar_wait(&bar[DRAIN], 0, a.wait_budget_ns);
            }
        } else if (warp == pv_warp) {
            // ---------------- PV issuer: [O_hi | O_lo] += V^T (MN-major) . [P_hi | P_lo]^T (MN-major)
            if (lane == 0) {
                // the hi (and lo) blocks that carry heads; N of an M = 128 product is at least 16
                constexpr int npv = C::p_terms * 8 * C::nb < 16 ? 16 : C::p_terms * 8 * C::nb;
                const uint32_t idesc_o = F8 ? umma_idesc_f16(kD, npv, 1, 1) : umma_idesc_bf16(kD, npv, 1, 1);
                int tcount = 0, icount = 0;
                bool ok = true;
                while (ok) {
                    const int slot = icount % kQD;
                    if (!wait_or_fail(&bar[I_FULL + slot], (icount / kQD) & 1, a, err)) break;
                    volatile int *q = queue + slot * 8;
                    const int t_begin = q[3], t_end = q[4];
                    mbar_arrive(&bar[I_EMPTY + slot]);
                    if (t_end < 0) break;
                    const int ntl = (t_end - t_begin + kTok - 1) / kTok;
                    const int ob = icount & 1;
                    if (icount >= 2 && !wait_or_fail(&bar[O_FREE + ob], ((icount >> 1) - 1) & 1, a, err)) break;
                    const uint32_t d_tmem = tO0 + ob * 2 * N;
                    for (int jj = 0; jj < ntl; ++jj) {
                        const int T = tcount + jj;
                        const int s = T % C::stages;
                        const int pb = T % C::pbufs;
                        if (!wait_or_fail(&bar[P_FULL + pb], (T / C::pbufs) & 1, a, err)) { ok = false; break; }
                        if (!wait_or_fail(&bar[(F8 ? VC_FULL : V_FULL) + s], (T / C::stages) & 1, a, err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t v_addr = smem_u32(smem + s * C::stage_bytes + (F8 ? 0 : kTile));
                        // one product of width 16 nb: the lo blocks follow the hi blocks at the same 2048-byte
                        // stride, so they are simply more columns
                        const uint32_t p_addr = smem_u32(ps + pb * 2 * C::p_half);
    #pragma unroll
                        for (int ks = 0; ks < kTok / 16; ++ks) {
                            // A = V^T: 16 tokens (two 8-row groups, 1024 B apart), 64-column blocks kHalf apart
                            // B = P^T: 16 tokens (two 128-byte core-matrix groups), 8-head blocks 2048 B apart
                            umma_ss(d_tmem, umma_smem_desc(v_addr + ks * 2048, kHalf, 1024, 2),
                                    umma_smem_desc(p_addr + ks * 256, 128, 2048, 0), idesc_o, (jj > 0 || ks > 0) ? 1u : 0u);
                        }
                        umma_commit(&bar[P_FREE + pb]);
                        // the stage's keys were read by an S^T product that completed before this P existed
                        umma_commit(&bar[(F8 ? R_EMPTY : KV_EMPTY) + s]);
                    }
                    if (!ok) break;
                    umma_commit(&bar[O_FULL + ob]);
                    tcount += ntl;
                    ++icount;
                }
                umma_commit(&bar[DRAIN_PV]);
                mbar_wait(&bar[DRAIN_PV], 0, a.wait_budget_ns);
            }
        }
    } else if (F8 && warp >= conv_warp0) {
        // ---------------- FP8 converter: thread ct owns token ct of each tile (TMEM lane ct of K)
        if constexpr (C::regsplit) set_max_regs<C::reg_conv, C::reg_launch>();
        const int ct = threadIdx.x - kWG * C::nwg;
        int tcount = 0, icount = 0;
        while (true) {
            const int slot = icount % kQD;
            if (!wait_or_fail(&bar[I_FULL + slot], (icount / kQD) & 1, a, err)) break;
            volatile int *qq = queue + slot * 8;
            const int t_begin = qq[3], t_end = qq[4];
            mbar_arrive(&bar[I_EMPTY + slot]);
            if (t_end < 0) break;
            // the group's query rows as two E4M3 terms of q 2^e per head (e putting the head's largest |q| in
            // [2^7, 2^8), below E4M3's largest 448): t0 = e4m3(v), t1 = e4m3(v - t0), the residual exact in
            // fp32.  A bf16 element v = m 2^(E-7) (m of 8 bits) leaves a residual k 2^(E-7) with |k| <= 8,
            // which E4M3 holds exactly while 2^(E-7) >= 2^-9, its subnormal step: every element down to 2^-10
            // of the head's largest is carried exactly, smaller ones within 2^-10 absolute (2^-17 of the
            // largest); the softmax undoes 2^e in its score factor.  The terms take the places of the row's
            // two bf16 halves, so B of S^T is the buffer read as 2N rows of 128 codes.
            const int qb = icount & 1;
            if (!wait_or_fail(&bar[Q_FULL + qb], (icount >> 1) & 1, a, err)) break;
            {
                constexpr int tpr = kWG / N;         // threads per query row (all in one warp)
                constexpr int cpt = 16 / tpr;        // 16-byte chunks per thread (16 per row: 2 halves x 8)
                const int row = ct / tpr, j0 = ct % tpr;
                uint8_t *qs = smem + C::q_off + qb * C::q_bytes;
                uint4 v[cpt];
                float mx = 0.f;
#pragma unroll
                for (int i = 0; i < cpt; ++i) {
                    const int k = j0 + i * tpr;
                    v[i] = *reinterpret_cast<const uint4 *>(qs + (k >> 3) * C::q_half + row * 128 + (k & 7) * 16);
                    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        mx = fmaxf(mx, fmaxf(fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e]))));
                }
#pragma unroll
                for (int o = tpr / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                const int ex = (int)((__float_as_uint(mx) >> 23) & 0xFF) - 127;
                const int e = min(7 - ex, 100);       // e in [-120, 100]: both 2^e and 2^-e are normal floats
                const float up = __uint_as_float((uint32_t)(127 + e) << 23);
                const float down = __uint_as_float((uint32_t)(127 - e) << 23);
                // every bf16 element of this row is in registers before any term overwrites the row
                __syncwarp();
#pragma unroll
                for (int i = 0; i < cpt; ++i) {
                    // physical chunk (k & 7) of half k >> 3 holds logical chunk l: elements 64 (k >> 3) + 8 l ..,
                    // which are codes 8 (l & 1) .. of logical code chunk 4 (k >> 3) + l / 2
                    const int k = j0 + i * tpr;
                    const int l = (k & 7) ^ (row & 7);
                    const int c = 4 * (k >> 3) + (l >> 1);
                    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                    float r[8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        r[2 * q] = bf16_lo(w[q]) * up;
                        r[2 * q + 1] = bf16_hi(w[q]) * up;
                    }
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt) {
                        uint32_t packed[2];
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            uint32_t code4 = 0;
#pragma unroll
                            for (int pr = 0; pr < 2; ++pr) {
                                const int e0 = 4 * q + 2 * pr;
                                uint16_t c2;
                                asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c2) : "f"(r[e0 + 1]), "f"(r[e0]));
                                uint32_t f2;   // the two codes back as f16 (exact), low element first
                                asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(f2) : "h"(c2));
                                r[e0] -= __half2float(__ushort_as_half((unsigned short)(f2 & 0xffffu)));
                                r[e0 + 1] -= __half2float(__ushort_as_half((unsigned short)(f2 >> 16)));
                                code4 |= (uint32_t)c2 << (16 * pr);
                            }
                            packed[q] = code4;
                        }
                        *reinterpret_cast<uint2 *>(qs + tt * C::q_half + row * 128 + ((c ^ (row & 7)) << 4) + (l & 1) * 8) =
                            make_uint2(packed[0], packed[1]);
                    }
                }
                if (j0 == 0) qfac[slot * N + row] = a.qk_factor * down;
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar[QC_FULL + qb]);
            mbar_arrive(&bar[QF_FULL + slot]);
            const int ntl = (t_end - t_begin + kTok - 1) / kTok;
            bool ok = true;
            for (int jj = 0; jj < ntl; ++jj) {
                const int T = tcount + jj;
                const int s = T % C::stages;
                if (!wait_or_fail(&bar[R_FULL + s], (T / C::stages) & 1, a, err)) { ok = false; break; }
                // the raw tiles were stored with the 128-byte swizzle: chunk c of row ct at c ^ (ct & 7)
                uint8_t *krow = smem + s * C::stage_bytes + ct * 128;
                // tokens past the piece's end may hold anything (NaN codes included): their values become
                // zeros, so that no 0 * NaN reaches an accumulator (their scores are masked by position)
                const bool valid = (t_begin + jj * kTok + ct) < t_end;
                // values -> f16 tile [2 halves][128 rows][128 B] with the 128-byte swizzle over the stage:
                // row ct of half 0 is where the key codes are (rewritten once the S^T products have read
                // them), row ct of half 1 where this thread's value codes are (read into registers first)
                uint4 vr[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) vr[c] = *reinterpret_cast<const uint4 *>(krow + kHalf + ((c ^ (ct & 7)) << 4));
                if (!wait_or_fail(&bar[K_READ + s], (T / C::stages) & 1, a, err)) { ok = false; break; }
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 lo4, hi4;
                    e4m3x4_to_f16x4(vr[c].x, lo4.x, lo4.y);
                    e4m3x4_to_f16x4(vr[c].y, lo4.z, lo4.w);
                    e4m3x4_to_f16x4(vr[c].z, hi4.x, hi4.y);
                    e4m3x4_to_f16x4(vr[c].w, hi4.z, hi4.w);
                    if (!valid) {
                        lo4 = make_uint4(0, 0, 0, 0);
                        hi4 = lo4;
                    }
                    const int j = 2 * (c & 3);   // 16 codes = two 16-byte f16 chunks of half c / 4
                    uint8_t *row = krow + (c >> 2) * kHalf;
                    *reinterpret_cast<uint4 *>(row + ((j ^ (ct & 7)) << 4)) = lo4;
                    *reinterpret_cast<uint4 *>(row + (((j + 1) ^ (ct & 7)) << 4)) = hi4;
                }
                fence_proxy_async_smem();
                mbar_arrive(&bar[VC_FULL + s]);
            }
            if (!ok) break;
            tcount += ntl;
            ++icount;
        }
    } else {
        // ---------------- softmax warpgroup wg: heads HW*wg .. HW*wg+HW-1; thread t owns token t of
        // each tile (TMEM lane t of S^T) and column d = t of O^T
        if constexpr (C::regsplit) set_max_regs<C::reg_soft, C::reg_launch>();
        const int wg = warp >> 2;
        const int quarter = warp & 3;              // TMEM lane quarter this warp may access
        const int t = quarter * 32 + lane;
        const int hs = wg * HW;                  // first head (column) of this warpgroup
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        volatile int *myvote = vote + wg * 8;
        int tcount = 0, icount = 0, uses = 0;
        bool ok = true;
        // The epilogue of a unit (its O^T from TMEM to the partials) runs after the next unit's first
        // tile, so that waiting for the unit's last PV product overlaps useful work.
        bool pend = false;
        int pb = 0, pkvh = 0, psplit = 0, pob = 0;   // psplit: piece index | pieces of the history << 16
        // FP8: O carries 128 p v_code; the value scale and 1/128 are applied here
        const float ofac = F8 ? a.o_factor : 1.f;
        auto epilogue = [&]() -> bool {
            if (!group_sync(&bar[GRP + wg], uses, a, err)) return false;      // lsum[pob] complete
            if (!wait_or_fail(&bar[O_FULL + pob], (((icount - 1) >> 1)) & 1, a, err)) return false;
            tc_fence_after();
            uint32_t o[HW], olo[HW];
            tmem_ldn<HW>(tO0 + pob * 2 * N + lane_off + hs, o);
            if constexpr (C::p_terms == 2) tmem_ldn<HW>(tO0 + pob * 2 * N + lane_off + 8 * C::nb + hs, olo);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < HW; ++h)
                o[h] = __float_as_uint((__uint_as_float(o[h]) + (C::p_terms == 2 ? __uint_as_float(olo[h]) : 0.f)) * ofac);
            const float *ls = lsum + pob * 4 * N;   // per-warp weight sums of the unit: [4][N]
            const int d = t;
            const size_t row0 = (size_t)pb * a.Hq + pkvh * g + hs;   // the warpgroup's first (b, query head) row
            if ((psplit >> 16) == 1) {
                // the whole history in one unit: normalise and write the output
#pragma unroll
                for (int h = 0; h < HW; ++h) {
                    if (hs + h >= g) break;
                    const float L = ls[hs + h] + ls[N + hs + h] + ls[2 * N + hs + h] + ls[3 * N + hs + h];
                    const float O = __uint_as_float(o[h]);
                    // a zero sum only for an empty history (output 0); a NaN sum (a NaN in the cache) stays NaN
                    a.out[(row0 + h) * kD + d] = __float2bfloat16_rn(L != 0.f ? O / L : 0.f);
                }
            } else {
                // one piece of several: a partial (o, m, l) for decode_combine_kernel
#pragma unroll
                for (int h = 0; h < HW; ++h) {
                    if (hs + h >= g) break;
                    a.part_o[((row0 + h) * a.nsplit + (psplit & 0xffff)) * kD + d] = __uint_as_float(o[h]);
                }
                // the (m, l) pairs: lane h of the warpgroup's first warp writes head h's, one store each
                if (quarter == 0 && lane < HW && hs + lane < g) {
                    const int hg = hs + lane;
                    const float mv = mst[pob * N + hg];
                    const float lv = ls[hg] + ls[N + hg] + ls[2 * N + hg] + ls[3 * N + hg];
                    *reinterpret_cast<float2 *>(a.part_ml + ((row0 + lane) * a.nsplit + (psplit & 0xffff)) * 2) =
                        make_float2(mv, lv);
                }
            }
            tc_fence_before();
            mbar_arrive(&bar[O_FREE + pob]);
            pend = false;
            return true;
        };
        while (ok) {
            const int slot = icount % kQD;
            if (!wait_or_fail(&bar[I_FULL + slot], (icount / kQD) & 1, a, err)) break;
            volatile int *qq = queue + slot * 8;
            const int b = qq[0], kvh = qq[1], split = qq[2], t_begin = qq[3], t_end = qq[4];
            if (t_end < 0) {
                mbar_arrive(&bar[I_EMPTY + slot]);
                if (pend) epilogue();   // the pending unit is icount - 1, as in the loop
                break;
            }
            // score factor per head: log2(e) * scale (FP8: times k_scale and the head's 2^-e, which the
            // converter leaves in the unit's slot; the slot is released only after reading them)
            float qf[HW];
            if constexpr (F8) {
                if (!wait_or_fail(&bar[QF_FULL + slot], (icount / kQD) & 1, a, err)) break;
#pragma unroll
                for (int h = 0; h < HW; ++h) qf[h] = qfac[slot * N + hs + h];
            } else {
#pragma unroll
                for (int h = 0; h < HW; ++h) qf[h] = a.qscale;
            }
            mbar_arrive(&bar[I_EMPTY + slot]);
            const int ntl = (t_end - t_begin + kTok - 1) / kTok;
            const int ob = icount & 1;
            float m_use[HW], l_part[HW];
#pragma unroll
            for (int h = 0; h < HW; ++h) {
                m_use[h] = -INFINITY;
                l_part[h] = 0.f;
            }
            for (int jj = 0; jj < ntl; ++jj) {
                const int T = tcount + jj;
                const int sb = T & 1;                  // vote and maxima buffers
                const int sbuf = T % C::sbufs;         // S buffer
                if (!wait_or_fail(&bar[S_FULL + sbuf], (T / C::sbufs) & 1, a, err)) { ok = false; break; }
                tc_fence_after();
                uint32_t raw[HW];
                tmem_ldn<HW>(tS0 + sbuf * C::s_cols + lane_off + hs, raw);
                if constexpr (F8) {
                    // the score is the sum of the products with the query's two terms
                    uint32_t raw1[HW];
                    tmem_ldn<HW>(tS0 + sbuf * C::s_cols + N + lane_off + hs, raw1);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < HW; ++h) raw[h] = __float_as_uint(__uint_as_float(raw[h]) + __uint_as_float(raw1[h]));
                }
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&bar[S_FREE + sbuf]);

                const bool valid = (t_begin + jj * kTok + t) < t_end;
                float x[HW];
                bool over = false;
#pragma unroll
                for (int h = 0; h < HW; ++h) {
                    x[h] = valid ? __uint_as_float(raw[h]) * qf[h] : -INFINITY;
                    over |= x[h] > m_use[h] + kMoveThreshold;
                }
                const int wflag = __any_sync(0xffffffffu, over) ? 1 : 0;
                if (lane == 0) myvote[sb * 4 + quarter] = wflag;
                if (!group_sync(&bar[GRP + wg], uses, a, err)) { ok = false; break; }
                const bool any_move = (myvote[sb * 4 + 0] | myvote[sb * 4 + 1] | myvote[sb * 4 + 2] |
                                       myvote[sb * 4 + 3]) != 0;
                float alpha[HW];
                bool rescale_o = false;
#pragma unroll
                for (int h = 0; h < HW; ++h) alpha[h] = 1.f;
                if (any_move) {
                    // this tile's maximum over all 128 tokens, per head
#pragma unroll
                    for (int h = 0; h < HW; ++h) {
                        float mx = x[h];
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                        if (lane == 0) red[(sb * 4 + quarter) * N + hs + h] = mx;
                    }
                    if (!group_sync(&bar[GRP + wg], uses, a, err)) { ok = false; break; }
#pragma unroll
                    for (int h = 0; h < HW; ++h) {
                        const float *rr = red + sb * 4 * N + hs + h;
                        const float tm = fmaxf(fmaxf(rr[0], rr[N]), fmaxf(rr[2 * N], rr[3 * N]));
                        const float m_new = fmaxf(m_use[h], tm);
                        if (m_new > m_use[h] + kMoveThreshold) {
                            alpha[h] = ex2(m_use[h] - m_new);     // 0 on the unit's first tile
                            m_use[h] = m_new;
                            l_part[h] *= alpha[h];
                            rescale_o = true;
                        }
                    }
                    rescale_o = rescale_o && (jj > 0);          // uniform: the warpgroup saw the same maxima
                }
                float p[HW];
#pragma unroll
                for (int h = 0; h < HW; ++h) {
                    p[h] = ex2(x[h] - m_use[h]);
                    l_part[h] += p[h];
                }
                // this tile's P buffer must have been read by its last PV product; a rescale of O also
                // needs the previous tile's PV finished
                const int pbuf = T % C::pbufs;
                if (T >= C::pbufs &&
                    !wait_or_fail(&bar[P_FREE + pbuf], ((T / C::pbufs) - 1) & 1, a, err)) { ok = false; break; }
                if (rescale_o && C::pbufs == 2 &&
                    !wait_or_fail(&bar[P_FREE + ((T - 1) & 1)], ((T - 1) >> 1) & 1, a, err)) { ok = false; break; }
                tc_fence_after();
                if (rescale_o) {
#pragma unroll
                    for (int part = 0; part < C::p_terms; ++part) {   // the hi (and the lo) columns
                        uint32_t o[HW];
                        tmem_ldn<HW>(tO0 + ob * 2 * N + lane_off + part * 8 * C::nb + hs, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < HW; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
                        tmem_stn<HW>(tO0 + ob * 2 * N + lane_off + part * 8 * C::nb + hs, o);
                    }
                    tmem_wait_st();
                }
                if constexpr (!F8) {
                    // Rows past the history may hold anything (NaN included) and the tensor cores would
                    // form 0 * NaN: in a partial tile the masked tokens zero their own V row once it has
                    // landed.  (The FP8 converter writes zeros for them instead.)
                    if (wg == 0 && t_end - (t_begin + jj * kTok) < kTok && !valid) {
                        const int st = T % C::stages;
                        if (!wait_or_fail(&bar[V_FULL + st], (T / C::stages) & 1, a, err)) { ok = false; break; }
                        uint8_t *vrow = smem + st * C::stage_bytes + kTile + t * 128;
                        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            *reinterpret_cast<uint4 *>(vrow + c * 16) = z;
                            *reinterpret_cast<uint4 *>(vrow + kHalf + c * 16) = z;
                        }
                    }
                }
                // P^T, MN-major without swizzle: core matrices of 8 tokens x 8 heads (128 B).  bf16: each
                // weight as hi plus lo = (p - hi), the lo blocks p_half after the hi ones; FP8: f16 of
                // 128 p alone (small weights stay normal).  With four heads only the first half of each
                // 16-byte core-matrix row is written: the other four columns of the products are never read.
                uint8_t *pdst = ps + pbuf * 2 * C::p_half + (t >> 3) * 128 + (t & 7) * 16;
#pragma unroll
                for (int hb = 0; hb < (HW + 7) / 8; ++hb) {
                    constexpr int E = HW < 8 ? HW / 2 : 4;   // packed pairs per block
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        if constexpr (F8) {
                            hi[e] = pack_f16x2(p[hb * 8 + 2 * e] * 128.f, p[hb * 8 + 2 * e + 1] * 128.f);
                        } else {
                            const float a0 = p[hb * 8 + 2 * e], a1 = p[hb * 8 + 2 * e + 1];
                            hi[e] = pack2(a0, a1);
                            lo[e] = pack2(a0 - bf16_lo(hi[e]), a1 - bf16_hi(hi[e]));
                        }
                    }
                    uint8_t *dst = pdst + (hs / 8 + hb) * 2048;
                    if constexpr (E == 4) {
                        *reinterpret_cast<uint4 *>(dst) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        if constexpr (C::p_terms == 2)
                            *reinterpret_cast<uint4 *>(dst + C::p_half) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    } else {
                        *reinterpret_cast<uint2 *>(dst) = make_uint2(hi[0], hi[1]);
                        if constexpr (C::p_terms == 2)
                            *reinterpret_cast<uint2 *>(dst + C::p_half) = make_uint2(lo[0], lo[1]);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar[P_FULL + pbuf]);
                // the previous unit's epilogue, now that its last PV has long been issued
                if (jj == 0 && pend && !epilogue()) { ok = false; break; }
            }
            if (!ok) break;
            // this unit's weight sums per head, reduced over each warp's 32 tokens; the CTA-wide sum is
            // finished in the (deferred) epilogue
#pragma unroll
            for (int h = 0; h < HW; ++h) {
                float v = l_part[h];
                v += __shfl_xor_sync(0xffffffffu, v, 16);
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                if (lane == 0) lsum[ob * 4 * N + quarter * N + hs + h] = v;
            }
            pend = true;
            pb = b;
            pkvh = kvh;
            psplit = split;
            pob = ob;
            // the maxima the unit's weights are relative to, for its (deferred) partial
            if (t == 0) {
#pragma unroll
                for (int h = 0; h < HW; ++h) mst[ob * N + hs + h] = m_use[h];
            }
            tcount += ntl;
            ++icount;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == mma_warp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::tmem_cols);
    }
}

template <int N, bool F8, int HW, int NWG>
cudaError_t launch_persistent(const CUtensorMap &tmK, const CUtensorMap &tmV, const CUtensorMap &tmQ,
                              const DecodeArgs &a, cudaStream_t stream)
{
    const int smem = TcCfg<N, F8, HW, NWG>::bytes;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(decode_persistent_kernel<N, F8, HW, NWG>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        if constexpr (TcCfg<N, F8, HW, NWG>::regsplit) {
            // setmaxnreg.inc waits until the decreases have freed enough of the registers the block was
            // launched with: refuse to launch unless the launch holds the whole split
            cudaFuncAttributes fa;
            if ((e = cudaFuncGetAttributes(&fa, decode_persistent_kernel<N, F8, HW, NWG>)) != cudaSuccess) return e;
            using Cf = TcCfg<N, F8, HW, NWG>;
            if ((long long)fa.numRegs * Cf::threads < (long long)kWG * (Cf::nwg * Cf::reg_soft + Cf::reg_conv + Cf::reg_last))
                return cudaErrorInvalidConfiguration;
        }
        attr_done[dev] = true;
    }
    // programmatic dependent launch: the prologue overlaps decode_plan_kernel (or, with the static
    // schedule, whatever ran before), which the kernel waits for (griddepcontrol.wait) before it
    // touches global memory
    cudaLaunchConfig_t cfg = {};
    const int units = a.B * a.Hkv;
    cfg.gridDim = dim3(a.static_plan && units < a.num_ctas ? units : a.num_ctas);
    cfg.blockDim = dim3(TcCfg<N, F8, HW, NWG>::threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_persistent_kernel<N, F8, HW, NWG>, tmK, tmV, tmQ, a);
}

}  // namespace

cudaError_t launch_decode_plan(const DecodeArgs &a, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(32);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_plan_kernel, a, a.num_ctas);
}

cudaError_t launch_decode_tc(const CUtensorMap &tmK, const CUtensorMap &tmV, const CUtensorMap &tmQ,
                             const DecodeArgs &a, cudaStream_t stream, bool fp8)
{
    if (fp8) {
        if (a.group <= 4) return launch_persistent<16, true, 4, 1>(tmK, tmV, tmQ, a, stream);
        if (a.group <= 8) return launch_persistent<16, true, 8, 1>(tmK, tmV, tmQ, a, stream);
        if (a.group <= 16) return launch_persistent<16, true, 8, 2>(tmK, tmV, tmQ, a, stream);
        if (a.group <= 32) return launch_persistent<32, true, 8, 4>(tmK, tmV, tmQ, a, stream);
        return cudaErrorInvalidValue;
    }
    if (a.group <= 4) return launch_persistent<16, false, 4, 1>(tmK, tmV, tmQ, a, stream);
    if (a.group <= 8) return launch_persistent<16, false, 8, 1>(tmK, tmV, tmQ, a, stream);
    if (a.group <= 16) return launch_persistent<16, false, 16, 1>(tmK, tmV, tmQ, a, stream);
    if (a.group <= 32) return launch_persistent<32, false, 16, 2>(tmK, tmV, tmQ, a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace gqa
