// ssm_scan_kernel.cuh -- warp-specialised selective-scan forward kernel for sm_100a.
//
// One thread block owns one group of CH = 32 channels of one sequence at a time
// and walks the item's time segment tile by tile (TT = 32 steps per tile). Nine
// warps with fixed roles, connected by mbarrier rings (every wait bounded in time
// and suspended in hardware while it waits):
//
//   C0..C3  consumers    the recurrence. Lane c is channel c of the group; warp w
//                        keeps states 4w .. 4w+3 of its lane's channel in registers.
//                        Per step a lane reads its channel's 8-byte record (u, Delta
//                        log2 e) and, with one warp-uniform broadcast load each, the
//                        B_t and C_t values of the warp's four states; it forms Abar,
//                        updates h = Abar h + u B and its partial readout sum_n C_n h_n
//                        (one 16-byte store per four steps).
//   P0, P1  prologue     per (t, channel), once: Delta = softplus(dt + bias), u =
//                        Delta x, Delta log2 e; widens the B and C rows to float32.
//                        P0 takes the first half of every tile's steps, P1 the second.
//   E0, E1  epilogue     per (t, channel): sums the four consumer partials, adds D x,
//                        applies the SiLU gate, rounds, and (E0) stores the y tile
//                        with TMA. Halves of the tile as for P.
//   L       loads        claims the (group, segment) items and streams x, dt, z, B, C
//                        of every tile with TMA into a STAGES-deep ring; a stage is
//                        refilled once both prologue and both epilogue warps have
//                        released it.
//
// Why this shape: shared memory delivers 128 bytes per clock per SM to registers,
// and a 16-byte load whose 32 lanes read different addresses costs four of those
// clocks, while one whose lanes all read the same address costs one. With lanes
// over channels and warps over states, B_t and C_t (shared by all channels) are
// warp-uniform, and the only lane-distinct data per step is the 8-byte record.
// Loops load all their shared-memory operands first and store last, so no store sits
// between a block's loads and the previous block's arithmetic; the consumers stage
// their arithmetic over blocks of four steps, while softplus and SiLU are evaluated
// value by value (staging those across many steps keeps too many special-function
// results in flight and measured 1.8x slower).
//
// Rings: stage (TMA, STAGES deep) -> P -> record ring (R_REC deep) -> consumers ->
// partial ring (R_PART deep) -> E, which also reads x and z from the stage. Between
// blocks, an item (group g, segment k) starts from the state its predecessor (g,
// k-1) published in the workspace.
//
// Short convolution (the CONV instantiations): the block's causal depthwise conv1d of
// width 4 and SiLU in front of the SSM, u_t = silu(cb + sum_k w_k x_{t-3+k}) (Mamba
// summary, block-architecture paragraph). The x box of every stage carries the three
// rows before the tile (TMA fills rows before t = 0 with zeros, or the prologue takes
// them from the caller's prefix). P evaluates u once per (t, channel), uses it for Delta
// u and writes it, in the token type, over the dt rows it has just read; E reads u there
// for D u in place of x. x still crosses HBM once.
//
// Exponentials: Abar_n = 2^(Delta log2 e * A[d,n]) on the SFU (ex2.approx). Where
// every row of A in the block is an arithmetic progression in n (A[d,n] = A[d,0] +
// n (A[d,1] - A[d,0]); the S4D-real rows A[d,n] = -(n+1) are one), a lane's four
// factors follow from two exponentials: Abar_{4w} and r = exp(Delta (A[d,1] -
// A[d,0])), then Abar_{4w+1} = Abar_{4w} r, Abar_{4w+2} = Abar_{4w} r^2,
// Abar_{4w+3} = Abar_{4w+1} r^2.
#pragma once

#include "../../include/ssm_scan.h"
#include "ssm_device.cuh"

namespace ssm {
namespace scan {

constexpr int CW = 4;                             // consumer warps (4 states each)
constexpr int NE = 2;                             // epilogue warps
constexpr int CH = 32;                            // channels per block (one per lane)
constexpr int WARP_P0 = CW;
constexpr int TT = 32;                            // time steps per tile
constexpr int TE = TT / NE;                       // steps per epilogue warp and tile
constexpr int KCONV = 4;                          // width of the short causal convolution
// Ring depths, blocks per SM and prologue warps. Shallow: 113 KB of shared memory (bf16),
// two blocks per SM. Deep: rings twice as deep, one block per SM; it decouples the roles
// further and is the better choice when there are too few channel groups to fill two
// blocks per SM (the long-context workload has 160 groups for 148 SMs). With the short
// convolution the prologue does about twice the work (the convolution and its SiLU), so
// the deep configuration spreads it over four prologue warps, one per SM sub-partition.
template <int STAGES_, int R_REC_, int R_PART_, int MINB_, int NP_ = 2>
struct Cfg {
    static constexpr int STAGES = STAGES_;  // TMA ring depth (tiles)
    static constexpr int R_REC = R_REC_;    // record ring depth
    static constexpr int R_PART = R_PART_;  // partial-sum ring depth
    static constexpr int MINB = MINB_;      // blocks per SM the registers are budgeted for
    static constexpr int NP = NP_;          // prologue warps
    static constexpr int TP = TT / NP;      // steps per prologue warp and tile
    static constexpr int WARP_E0 = CW + NP, WARP_L = CW + NP + NE;
    static constexpr int NTHREADS = (CW + NP + NE + 1) * 32;
    static_assert(TP % 8 == 0, "a prologue warp takes whole pairs of steps and whole 16-byte B/C chunks");
};
#ifndef SSM_DEEP_STAGES
#define SSM_DEEP_STAGES 8
#endif
#ifndef SSM_DEEP_REC
#define SSM_DEEP_REC 4
#endif
#ifndef SSM_DEEP_PART
#define SSM_DEEP_PART 4
#endif
using Shallow = Cfg<6, 2, 2, 2>;
using Deep = Cfg<SSM_DEEP_STAGES, SSM_DEEP_REC, SSM_DEEP_PART, 1>;
using DeepConv = Cfg<SSM_DEEP_STAGES, SSM_DEEP_REC, SSM_DEEP_PART, 1, 4>;
constexpr int YBUF = 3;                           // y staging buffers for the TMA store
constexpr int kMaxN = 16;                         // state slots per channel
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // every device-side wait gives up after 2 s
constexpr uint32_t kSuspendNs = 20000;            // hardware suspend hint per try_wait

enum : int { F_FIRST = 1, F_LAST = 2, F_END = 4, F_STRUCT = 8 };

struct TileMeta {
    long long g, k;  // channel group and time segment of the tile's item
    int b, d0;       // the group's sequence and first channel (divided out once per item)
    int t0, tlen;    // first step of the tile and its number of valid steps
    int flags;       // F_FIRST | F_LAST | F_END | F_STRUCT
    int j;           // tile index inside the item
};

struct Params {
    int64_t Bsz, L, D, N;
    int64_t G, Dg, K, seg_len, items;
    const void *Bm;
    const void *Cm;
    const float *A;
    const float *Dskip;
    const float *dt_bias;
    const float *h0;
    float *h_last;
    uint32_t *counter;
    uint32_t *status;
    uint32_t *flags;
    float *carry;
    const float *conv_w;  // [D, 4] taps of the short convolution (CONV instantiations)
    const float *conv_b;  // [D] or null
    const void *conv_x0;  // [B, 3, D] tokens before t = 0, or null for zeros
    int has_gate, softplus, allow_structured, drop_handoff, bc_tma;
    // Sequence-parallel evaluation (kModeHandoff: segment k waits for k-1's state):
    // kModeLocal: every segment runs from a zero state (segment 0 from h0, so its outputs
    // are final and only its y is stored), writes its end state to seg_local and its sum of
    // Delta log2 e per channel to seg_dsum; kModeFromCarry: segments 1 .. K-1 (the items
    // from item_base = G on) start from seg_state (the combine kernel's result).
    int mode;
    int64_t item_base;  // the first item this launch claims
    float *seg_local;  // [G K][CW][CH] float4
    float *seg_state;  // [G K][CW][CH] float4
    float *seg_dsum;   // [G K][4 prologue slots][CH]
};
enum : int { kModeHandoff = 0, kModeLocal = 1, kModeFromCarry = 2 };

template <typename T, typename C, bool CONV = false>
struct Layout {
    static constexpr int STAGES = C::STAGES, R_REC = C::R_REC, R_PART = C::R_PART;
    static constexpr int BOX = TT * CH;           // elements of one token box [TT][CH]
    static constexpr int BCBOX = TT * kMaxN;      // elements of one B or C box [TT][16]
    static constexpr int HALO = CONV ? KCONV - 1 : 0;  // rows of x before the tile in its box
    static constexpr size_t tok_bytes = size_t(BOX) * sizeof(T);
    static constexpr size_t bc_bytes = size_t(BCBOX) * sizeof(T);
    static constexpr size_t xbox_bytes = size_t(TT + HALO) * CH * sizeof(T);  // what one x box delivers
    static constexpr size_t x_bytes = (xbox_bytes + 127) / 128 * 128;
    // stage: x (with its halo rows) | dt | z | B | C
    static constexpr size_t st_x = 0, st_dt = x_bytes, st_z = x_bytes + tok_bytes, st_b = x_bytes + 2 * tok_bytes,
                            st_c = x_bytes + 2 * tok_bytes + bc_bytes;
    static constexpr size_t stage_bytes = x_bytes + 2 * tok_bytes + 2 * bc_bytes;
    static constexpr size_t stage_off = 0;
    static constexpr size_t rec_off = stage_off + STAGES * stage_bytes;
    static constexpr size_t rec_bytes = size_t(BOX) * 8;            // float4 (u, Delta log2 e) x 2 per (t pair, c)
    static constexpr size_t bcf_off = rec_off + R_REC * rec_bytes;
    static constexpr size_t bcf_bytes = size_t(TT) * 32 * 4;        // [TT][B 16 | C 16] float
    static constexpr size_t part_off = bcf_off + R_REC * bcf_bytes;
    static constexpr size_t part_bytes = size_t(CW) * (TT / 4) * CH * 16;  // [w][t/4][c] float4
    static constexpr size_t yout_off = part_off + R_PART * part_bytes;
    static constexpr size_t yout_bytes = tok_bytes;
    static constexpr size_t smeta_off = yout_off + YBUF * yout_bytes;
    static constexpr size_t tmeta_off = smeta_off + STAGES * sizeof(TileMeta);
    static constexpr size_t bar_off = (tmeta_off + R_REC * sizeof(TileMeta) + 15) / 16 * 16;
    static constexpr int NBARS = 2 * STAGES + 2 * R_REC + 2 * R_PART;
    static constexpr size_t total = bar_off + NBARS * 8;
    static_assert(stage_bytes % 128 == 0 && tok_bytes % 128 == 0 && bc_bytes % 128 == 0,
                  "TMA boxes must stay 128-byte aligned");
    static_assert(rec_off % 128 == 0 && yout_off % 128 == 0, "TMA/vector buffers must stay aligned");
};

// Bounded wait for the completion of phase `parity` of an mbarrier by every lane of
// a warp; each try suspends the lane in hardware (up to kSuspendNs) instead of
// spinning. Warp-uniform answer: false if the limit was reached.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity) {
    bool ok = mbar_try_wait_suspend(bar, parity);
    if (!ok) {
        const uint64_t start = globaltimer_ns();
        while (!(ok = mbar_try_wait_suspend(bar, parity)))
            if (globaltimer_ns() - start > kWaitLimitNs) break;
    }
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One arrival per warp: the warp's shared-memory accesses are ordered before lane 0's
// release-arrive by __syncwarp (a 32-lane arrive costs the shared-memory pipe far more).
__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ void consumer_sync() {  // named barrier 1: the consumer warps only
    asm volatile("bar.sync 1, %0;" ::"n"(CW * 32) : "memory");
}
__device__ __forceinline__ void epilogue_sync() {  // named barrier 2: the epilogue warps only
    asm volatile("bar.sync 2, %0;" ::"n"(NE * 32) : "memory");
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

__device__ __forceinline__ void set_timeout(uint32_t *status, int lane) {
    if (lane == 0) atomicExch(status, uint32_t(SSM_ERR_TIMEOUT));
}

// Exact zero-order hold for two states: w = Bbar / B per unit input = (Abar - 1) / A,
// with z = Delta A; below |z| = 1/16 the series Delta (1 + z/2 + z^2/6 + z^3/24 +
// z^4/120) (truncation below 2e-9 relative), where Abar - 1 would lose precision.
// a: Abar; ia: 1/A (0 where A = 0, where the series gives Delta).
__device__ __forceinline__ float2 zoh_weight(const float2 z, const float2 a, const float2 ia, const float delta) {
    float2 q = __ffma2_rn(z, f2(1.f / 120.f, 1.f / 120.f), f2(1.f / 24.f, 1.f / 24.f));
    q = __ffma2_rn(z, q, f2(1.f / 6.f, 1.f / 6.f));
    q = __ffma2_rn(z, q, f2(0.5f, 0.5f));
    q = __ffma2_rn(z, q, f2(1.f, 1.f));
    const float2 ser = __fmul2_rn(f2(delta, delta), q);
    const float2 dir = __fmul2_rn(__fadd2_rn(a, f2(-1.f, -1.f)), ia);
    return f2(fabsf(z.x) < 0.0625f ? ser.x : dir.x, fabsf(z.y) < 0.0625f ? ser.y : dir.y);
}

// ---------------------------------------------------------------- consumers
// One block of four steps for one lane: the factors Abar and the inputs u B of the
// warp's four states (pairs 01 and 23) from the block's records (two steps each) and B
// rows.
template <bool STRUCT, bool ZOH>
__device__ __forceinline__ void block_factors(const float4 r0, const float4 r1, const float4 (&b4)[4], const float4 Aq,
                                              const float del, const float4 zA, const float4 iA, float2 (&a01)[4],
                                              float2 (&a23)[4], float2 (&ub01)[4], float2 (&ub23)[4]) {
    constexpr int S = 4;
    const float2 p[S] = {f2(r0.x, r0.y), f2(r0.z, r0.w), f2(r1.x, r1.y), f2(r1.z, r1.w)};
    if (STRUCT) {
        float2 x[S];
#pragma unroll
        for (int s = 0; s < S; ++s) x[s] = __fmul2_rn(f2(p[s].y, p[s].y), f2(Aq.x, del));
        float a0[S], r[S];
#pragma unroll
        for (int s = 0; s < S; ++s) {
            a0[s] = ex2_approx(x[s].x);
            r[s] = ex2_approx(x[s].y);
        }
#pragma unroll
        for (int s = 0; s < S; ++s) a01[s] = f2(a0[s], a0[s] * r[s]);
#pragma unroll
        for (int s = 0; s < S; ++s) a23[s] = __fmul2_rn(a01[s], f2(r[s] * r[s], r[s] * r[s]));
    } else {
        float2 x01[S], x23[S];
#pragma unroll
        for (int s = 0; s < S; ++s) {
            x01[s] = __fmul2_rn(f2(p[s].y, p[s].y), f2(Aq.x, Aq.y));
            x23[s] = __fmul2_rn(f2(p[s].y, p[s].y), f2(Aq.z, Aq.w));
        }
#pragma unroll
        for (int s = 0; s < S; ++s) {
            a01[s] = f2(ex2_approx(x01[s].x), ex2_approx(x01[s].y));
            a23[s] = f2(ex2_approx(x23[s].x), ex2_approx(x23[s].y));
        }
    }
#pragma unroll
    for (int s = 0; s < S; ++s) {
        ub01[s] = __fmul2_rn(f2(p[s].x, p[s].x), f2(b4[s].x, b4[s].y));
        ub23[s] = __fmul2_rn(f2(p[s].x, p[s].x), f2(b4[s].z, b4[s].w));
    }
    if (ZOH) {  // the record carries x; Bbar x = B x (Abar - 1) / A
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const float delta = p[s].y * kLn2;
            const float2 z01 = __fmul2_rn(f2(p[s].y, p[s].y), f2(zA.x, zA.y));
            const float2 z23 = __fmul2_rn(f2(p[s].y, p[s].y), f2(zA.z, zA.w));
            ub01[s] = __fmul2_rn(ub01[s], zoh_weight(z01, a01[s], f2(iA.x, iA.y), delta));
            ub23[s] = __fmul2_rn(ub23[s], zoh_weight(z23, a23[s], f2(iA.z, iA.w), delta));
        }
    }
}

// The recurrence of one block of four steps and the partial readout over the warp's
// four states, the last additions of two steps paired; returns the four partials.
__device__ __forceinline__ float4 block_recur(const float2 (&a01)[4], const float2 (&a23)[4], const float2 (&ub01)[4],
                                              const float2 (&ub23)[4], const float4 (&c4)[4], float2 &h01, float2 &h23) {
    constexpr int S = 4;
    float2 q[S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
        h01 = __ffma2_rn(a01[s], h01, ub01[s]);
        h23 = __ffma2_rn(a23[s], h23, ub23[s]);
        q[s] = __ffma2_rn(f2(c4[s].z, c4[s].w), h23, __fmul2_rn(f2(c4[s].x, c4[s].y), h01));
    }
    const float2 y01 = __fadd2_rn(f2(q[0].x, q[1].x), f2(q[0].y, q[1].y));
    const float2 y23 = __fadd2_rn(f2(q[2].x, q[3].x), f2(q[2].y, q[3].y));
    return make_float4(y01.x, y01.y, y23.x, y23.y);
}

// TT steps of one tile for one lane (its channel, the warp's four states), in blocks of
// four steps, software-pipelined: the shared-memory operands of a block are loaded
// LOOK blocks ahead of its recurrence and, with AHEAD, its factors (the exponentials and
// u B) are formed one block ahead, so that the latency of the loads and of the
// special-function unit overlaps the recurrence of the block before. rec: this lane's
// records, one float4 (u, Delta log2 e) x 2 per two steps (stride CH); bc: B of the
// warp's states (stride 32 floats per step; C at +16); part: this lane's partials
// (stride CH float4 per block of four steps). Aq: A[c][4w .. 4w+3]; del: A[c][1] -
// A[c][0]; ZOH (exact zero-order hold): zA = A ln 2 and iA = 1/A of the four states, and
// the records carry x in place of Delta x.
template <bool STRUCT, bool ZOH, bool AHEAD>
__device__ __forceinline__ void consume_tile(const float4 *__restrict__ rec, const float *__restrict__ bc,
                                             float4 *__restrict__ part, const float4 Aq, const float del,
                                             const float4 zA, const float4 iA, float2 &h01, float2 &h23) {
    constexpr int S = 4, NB = TT / S;
    auto load = [&](int blk, float4 &r0, float4 &r1, float4 (&b4)[S], float4 (&c4)[S]) {
        r0 = rec[(2 * blk) * CH];
        r1 = rec[(2 * blk + 1) * CH];
#pragma unroll
        for (int s = 0; s < S; ++s) {
            b4[s] = *reinterpret_cast<const float4 *>(bc + (blk * S + s) * 32);  // warp-uniform
            c4[s] = *reinterpret_cast<const float4 *>(bc + (blk * S + s) * 32 + 16);
        }
    };
    if (AHEAD) {
        float4 r0, r1, b4[S], c4[S], rn0, rn1, bn[S], cn[S];
        float2 a01[S], a23[S], ub01[S], ub23[S];
        float4 cc[S];  // C rows of the block whose factors are in a01 .. ub23
        load(0, r0, r1, b4, c4);
        block_factors<STRUCT, ZOH>(r0, r1, b4, Aq, del, zA, iA, a01, a23, ub01, ub23);
#pragma unroll
        for (int s = 0; s < S; ++s) cc[s] = c4[s];
        load(1, rn0, rn1, bn, cn);
#pragma unroll
        for (int blk = 0; blk < NB; ++blk) {
            float2 na01[S], na23[S], nub01[S], nub23[S];
            float4 ncc[S];
            if (blk + 1 < NB) {  // factors of the next block (its operands were loaded last time)
                block_factors<STRUCT, ZOH>(rn0, rn1, bn, Aq, del, zA, iA, na01, na23, nub01, nub23);
#pragma unroll
                for (int s = 0; s < S; ++s) ncc[s] = cn[s];
            }
            if (blk + 2 < NB) load(blk + 2, rn0, rn1, bn, cn);
            part[blk * CH] = block_recur(a01, a23, ub01, ub23, cc, h01, h23);
            if (blk + 1 < NB) {
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    a01[s] = na01[s];
                    a23[s] = na23[s];
                    ub01[s] = nub01[s];
                    ub23[s] = nub23[s];
                    cc[s] = ncc[s];
                }
            }
        }
    } else {
        float4 r0, r1, b4[S], c4[S], rn0, rn1, bn[S], cn[S];
        load(0, r0, r1, b4, c4);
#pragma unroll
        for (int blk = 0; blk < NB; ++blk) {
            if (blk + 1 < NB) load(blk + 1, rn0, rn1, bn, cn);
            float2 a01[S], a23[S], ub01[S], ub23[S];
            block_factors<STRUCT, ZOH>(r0, r1, b4, Aq, del, zA, iA, a01, a23, ub01, ub23);
            part[blk * CH] = block_recur(a01, a23, ub01, ub23, c4, h01, h23);
            if (blk + 1 < NB) {
                r0 = rn0;
                r1 = rn1;
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    b4[s] = bn[s];
                    c4[s] = cn[s];
                }
            }
        }
    }
}

// ------------------------------------------------------ short convolution
// u for rows t0 .. t0+2*NPR-1 of a tile, as pairs: u_t = silu(cb + w.x x_{t-3} + w.y
// x_{t-2} + w.z x_{t-1} + w.w x_t). sx points at row 0 of the tile; the three rows before
// it are the box's halo. With use_x0 (the sequence's first rows, t0 = 0) the caller's
// prefix x0 replaces the halo rows, which TMA filled with zeros.
template <typename T, int NPR>
__device__ __forceinline__ void conv_silu_rows(const T *__restrict__ sx, const int t0, const float4 w, const float cb,
                                               const bool use_x0, const float3 x0, float2 (&u)[NPR]) {
    constexpr int NR = 2 * NPR + KCONV - 1;
    float r[NR];
#pragma unroll
    for (int j = 0; j < NR; ++j) r[j] = Tok<T>::to_f(sx[(t0 - (KCONV - 1) + j) * CH]);
    if (use_x0) {
        r[0] = x0.x;
        r[1] = x0.y;
        r[2] = x0.z;
    }
#pragma unroll
    for (int q = 0; q < NPR; ++q) {
        float2 v = __ffma2_rn(f2(w.x, w.x), f2(r[2 * q], r[2 * q + 1]), f2(cb, cb));
        v = __ffma2_rn(f2(w.y, w.y), f2(r[2 * q + 1], r[2 * q + 2]), v);
        v = __ffma2_rn(f2(w.z, w.z), f2(r[2 * q + 2], r[2 * q + 3]), v);
        v = __ffma2_rn(f2(w.w, w.w), f2(r[2 * q + 3], r[2 * q + 4]), v);
        u[q] = f2(silu_f(v.x), silu_f(v.y));  // per value, as softplus and the gate
    }
}

// Taps and bias of the short convolution for channel d (zeros past the last channel).
__device__ __forceinline__ void load_conv(const Params &p, const int64_t d, float4 &w, float &b) {
    const bool ok = d < p.D;
    w = ok ? __ldg(reinterpret_cast<const float4 *>(p.conv_w) + d) : make_float4(0.f, 0.f, 0.f, 0.f);
    b = (ok && p.conv_b) ? __ldg(p.conv_b + d) : 0.f;
}

// The caller's three tokens before t = 0 for channel d of sequence b, oldest first; false
// (the halo keeps TMA's zeros) without a prefix or past the last channel.
template <typename T>
__device__ __forceinline__ bool conv_prefix(const Params &p, const int64_t b, const int64_t d, float3 &x0) {
    if (!p.conv_x0 || d >= p.D) return false;
    const T *src = static_cast<const T *>(p.conv_x0) + b * (KCONV - 1) * p.D + d;
    x0 = make_float3(Tok<T>::ldg(src), Tok<T>::ldg(src + p.D), Tok<T>::ldg(src + 2 * p.D));
    return true;
}

// ---------------------------------------------------------------- prologue
// Records of TP steps (rows t0 .. t0+TP-1 of a tile) for channel c: (u = Delta x,
// Delta log2 e), with Delta = softplus(dt + bias) (or dt + bias); with `zoh` (exact
// zero-order hold) u = x, the consumers apply the weight. Rows at or past tlen get
// (0, 0): Abar = 1, no input. CONV: x is the short convolution's output (cw, cb, and
// use_x0 / x0 as for conv_silu_rows), which is also written over the dt rows read.
// DSUM: returns the sum of the valid rows' Delta log2 e (else 0).
template <typename T, bool CONV, int TP, bool DSUM>
__device__ __forceinline__ float prologue_rows(const T *__restrict__ sx, T *__restrict__ sdt,
                                              float4 *__restrict__ rec, const int t0, const int tlen,
                                              const float bias, const bool softplus, const bool zoh,
                                              const float4 cw, const float cb, const bool use_x0, const float3 x0) {
    constexpr int NPR = TP / 2;  // pairs of steps
    float2 v[NPR], xv[NPR];
#pragma unroll
    for (int q = 0; q < NPR; ++q) {
        const int t = t0 + 2 * q;
        v[q] = f2(Tok<T>::to_f(sdt[t * CH]), Tok<T>::to_f(sdt[(t + 1) * CH]));
        if (!CONV) xv[q] = f2(Tok<T>::to_f(sx[t * CH]), Tok<T>::to_f(sx[(t + 1) * CH]));
    }
    if (CONV) conv_silu_rows<T, NPR>(sx, t0, cw, cb, use_x0, x0, xv);
#pragma unroll
    for (int q = 0; q < NPR; ++q) v[q] = __fadd2_rn(v[q], f2(bias, bias));
    // softplus per value (measured: 1.8x faster here than the same arithmetic staged
    // across all pairs, which keeps too many SFU results in flight)
    float2 delta[NPR];
#pragma unroll
    for (int q = 0; q < NPR; ++q)
        delta[q] = softplus ? f2(softplus_f(v[q].x), softplus_f(v[q].y)) : v[q];
    float2 u[NPR], dl[NPR];
    float dsum = 0.f;  // sum of the valid rows' Delta log2 e (the sequence-parallel local pass)
#pragma unroll
    for (int q = 0; q < NPR; ++q) {
        u[q] = zoh ? xv[q] : __fmul2_rn(delta[q], xv[q]);
        dl[q] = __fmul2_rn(delta[q], f2(kLog2e, kLog2e));
    }
#pragma unroll
    for (int q = 0; q < NPR; ++q) {
        const int t = t0 + 2 * q;
        const bool v0 = t < tlen, v1 = t + 1 < tlen;
        rec[(t / 2) * CH] = make_float4(v0 ? u[q].x : 0.f, v0 ? dl[q].x : 0.f, v1 ? u[q].y : 0.f, v1 ? dl[q].y : 0.f);
        if (DSUM) dsum += (v0 ? dl[q].x : 0.f) + (v1 ? dl[q].y : 0.f);
    }
    if (CONV) {  // the epilogue's D u
#pragma unroll
        for (int q = 0; q < NPR; ++q) {
            const int t = t0 + 2 * q;
            sdt[t * CH] = Tok<T>::from_f(xv[q].x);
            sdt[(t + 1) * CH] = Tok<T>::from_f(xv[q].y);
        }
    }
    return dsum;
}

// ---------------------------------------------------------------- epilogue
// y for TE steps (rows t0 .. t0+TE-1) of channel c: sum of the four consumer
// partials, + D x, times silu(z), rounded to T. (With the short convolution sx points
// at the u rows the prologue wrote.)
template <typename T>
__device__ __forceinline__ void epilogue_rows(const float4 *__restrict__ part, const T *__restrict__ sx,
                                              const T *__restrict__ sz, T *__restrict__ yo, const int t0,
                                              const float dd, const bool gate) {
    constexpr int NB = TE / 4;  // blocks of four steps
    float2 y01[NB], y23[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const int blk = t0 / 4 + b;
        float4 v[CW];
#pragma unroll
        for (int w = 0; w < CW; ++w) v[w] = part[(w * (TT / 4) + blk) * CH];
        float2 lo = __fadd2_rn(f2(v[0].x, v[0].y), f2(v[1].x, v[1].y));
        float2 hi = __fadd2_rn(f2(v[0].z, v[0].w), f2(v[1].z, v[1].w));
        const float2 lo2 = __fadd2_rn(f2(v[2].x, v[2].y), f2(v[3].x, v[3].y));
        const float2 hi2 = __fadd2_rn(f2(v[2].z, v[2].w), f2(v[3].z, v[3].w));
        lo = __fadd2_rn(lo, lo2);
        hi = __fadd2_rn(hi, hi2);
        const int t = t0 + 4 * b;
        const float2 x01 = f2(Tok<T>::to_f(sx[t * CH]), Tok<T>::to_f(sx[(t + 1) * CH]));
        const float2 x23 = f2(Tok<T>::to_f(sx[(t + 2) * CH]), Tok<T>::to_f(sx[(t + 3) * CH]));
        y01[b] = __ffma2_rn(f2(dd, dd), x01, lo);
        y23[b] = __ffma2_rn(f2(dd, dd), x23, hi);
    }
    if (gate) {
        // silu(z) = z / (1 + e^-z), per value (as for softplus in the prologue)
        float2 z01[NB], z23[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int t = t0 + 4 * b;
            z01[b] = f2(Tok<T>::to_f(sz[t * CH]), Tok<T>::to_f(sz[(t + 1) * CH]));
            z23[b] = f2(Tok<T>::to_f(sz[(t + 2) * CH]), Tok<T>::to_f(sz[(t + 3) * CH]));
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            y01[b] = __fmul2_rn(y01[b], f2(silu_f(z01[b].x), silu_f(z01[b].y)));
            y23[b] = __fmul2_rn(y23[b], f2(silu_f(z23[b].x), silu_f(z23[b].y)));
        }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const int t = t0 + 4 * b;
        yo[t * CH] = Tok<T>::from_f(y01[b].x);
        yo[(t + 1) * CH] = Tok<T>::from_f(y01[b].y);
        yo[(t + 2) * CH] = Tok<T>::from_f(y23[b].x);
        yo[(t + 3) * CH] = Tok<T>::from_f(y23[b].y);
    }
}

// ------------------------------------------------------------------- kernel
// SEQ: the sequence-parallel passes (p.mode kModeLocal or kModeFromCarry); the hand-off
// kernel (SEQ false) carries none of their code.
template <typename T, typename C, bool ZOH, bool CONV, bool SEQ = false>
__global__ void __launch_bounds__(C::NTHREADS, C::MINB)
    scan_ws_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_dt,
                   const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                   const Params p) {
    using S = Layout<T, C, CONV>;
    constexpr int STAGES = C::STAGES, R_REC = C::R_REC, R_PART = C::R_PART;
    constexpr int NP = C::NP, TP = C::TP, WARP_E0 = C::WARP_E0, WARP_L = C::WARP_L;
    extern __shared__ __align__(1024) unsigned char smem[];
    TileMeta *smeta = reinterpret_cast<TileMeta *>(smem + S::smeta_off);  // per stage
    TileMeta *tmeta = reinterpret_cast<TileMeta *>(smem + S::tmeta_off);  // per record slot
    uint64_t *bar_full = reinterpret_cast<uint64_t *>(smem + S::bar_off);
    uint64_t *bar_sfree = bar_full + STAGES;
    uint64_t *bar_rec_full = bar_sfree + STAGES;
    uint64_t *bar_rec_free = bar_rec_full + R_REC;
    uint64_t *bar_part_full = bar_rec_free + R_REC;
    uint64_t *bar_part_free = bar_part_full + R_PART;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&bar_full[s], 1);
            mbar_init(&bar_sfree[s], NP + NE);
        }
        for (int r = 0; r < R_REC; ++r) {
            mbar_init(&bar_rec_full[r], NP);
            mbar_init(&bar_rec_free[r], CW);
        }
        for (int r = 0; r < R_PART; ++r) {
            mbar_init(&bar_part_full[r], CW);
            mbar_init(&bar_part_free[r], NE);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == WARP_L) {
        // ================================================================ L: loads
        const uint32_t tx_bytes =
            uint32_t(S::xbox_bytes + (p.has_gate ? 2 : 1) * S::tok_bytes + (p.bc_tma ? 2 * S::bc_bytes : 0));
        if (lane == 0) {
            prefetch_tensormap(&tm_x);
            prefetch_tensormap(&tm_dt);
            if (p.has_gate) prefetch_tensormap(&tm_z);
            if (p.bc_tma) {
                prefetch_tensormap(&tm_b);
                prefetch_tensormap(&tm_c);
            }
        }
        long long li_g = 0, li_k = 0, li_beg = 0, li_end = 0;
        int li_j = 0, li_n = 0, li_b = 0, li_d0 = 0;
        bool li_ok = false;
        auto claim = [&]() {
            unsigned int it = 0;
            if (lane == 0) it = atomicAdd(p.counter, 1u);
            it = __shfl_sync(0xffffffffu, it, 0);
            if (SEQ) it += (unsigned int)p.item_base;
            li_ok = (long long)it < p.items;
            if (li_ok) {
                li_k = (long long)it / p.G;
                li_g = (long long)it % p.G;
                li_b = int(li_g / p.Dg);
                li_d0 = int((li_g - (long long)li_b * p.Dg) * CH);
                li_beg = li_k * p.seg_len;
                li_end = min((long long)p.L, li_beg + p.seg_len);
                li_n = int((li_end - li_beg + TT - 1) / TT);
                li_j = 0;
            }
        };
        claim();
        for (int i = 0;; ++i) {
            const int st = i % STAGES;
            if (i >= STAGES && !warp_wait(&bar_sfree[st], uint32_t(i / STAGES - 1) & 1u)) {
                set_timeout(p.status, lane);
                break;
            }
            TileMeta m;
            m.g = li_g;
            m.b = li_b;
            m.d0 = li_d0;
            m.k = li_k;
            m.j = li_j;
            m.t0 = int(li_beg + (long long)li_j * TT);
            m.tlen = int(li_end - m.t0 < TT ? li_end - m.t0 : TT);
            m.flags = li_ok ? ((li_j == 0 ? F_FIRST : 0) | (li_j == li_n - 1 ? F_LAST : 0)) : F_END;
            if (lane == 0) {
                smeta[st] = m;
                if (li_ok) {
                    unsigned char *stage = smem + S::stage_off + size_t(st) * S::stage_bytes;
                    const int b = m.b, d0 = m.d0;
                    mbar_arrive_expect_tx(&bar_full[st], tx_bytes);
                    // CONV: the box starts HALO rows early (before t = 0 TMA reads zeros)
                    tma_load_3d(stage + S::st_x, &tm_x, &bar_full[st], d0, m.t0 - S::HALO, b);
                    tma_load_3d(stage + S::st_dt, &tm_dt, &bar_full[st], d0, m.t0, b);
                    if (p.has_gate) tma_load_3d(stage + S::st_z, &tm_z, &bar_full[st], d0, m.t0, b);
                    if (p.bc_tma) {
                        tma_load_3d(stage + S::st_b, &tm_b, &bar_full[st], 0, m.t0, b);
                        tma_load_3d(stage + S::st_c, &tm_c, &bar_full[st], 0, m.t0, b);
                    }
                } else {
                    mbar_arrive(&bar_full[st]);  // end of the stream: complete the phase without data
                }
            }
            __syncwarp();
            if (!li_ok) break;
            if (++li_j == li_n) claim();
        }
    } else if (warp >= WARP_E0) {
        // ================================================================ E: epilogue
        const int h = warp - WARP_E0;
        const int c = lane;
        float dd = 0.f;
        for (int i = 0;; ++i) {
            const int pr = i % R_PART, st = i % STAGES;
            if (!warp_wait(&bar_part_full[pr], uint32_t(i / R_PART) & 1u)) {
                set_timeout(p.status, lane);
                break;
            }
            const TileMeta m = smeta[st];
            if (m.flags & F_END) break;
            if (!warp_wait(&bar_full[st], uint32_t(i / STAGES) & 1u)) {
                set_timeout(p.status, lane);
                break;
            }
            if (m.flags & F_FIRST) {
                const int64_t d = m.d0 + c;
                dd = (d < p.D && p.Dskip) ? __ldg(p.Dskip + d) : 0.f;
            }
            const unsigned char *stage = smem + S::stage_off + size_t(st) * S::stage_bytes;
            // the SSM's input: x, or the short convolution's u that P left in the dt rows
            const T *sx = reinterpret_cast<const T *>(stage + (CONV ? S::st_dt : S::st_x)) + c;
            const T *sz = reinterpret_cast<const T *>(stage + S::st_z) + c;
            const float4 *part = reinterpret_cast<const float4 *>(smem + S::part_off + pr * S::part_bytes) + c;
            T *yo = reinterpret_cast<T *>(smem + S::yout_off + (i % YBUF) * S::yout_bytes) + c;
            // (the local pass keeps the y of segment 0 only: the other segments' tiles pass through)
            if (!SEQ || p.mode != kModeLocal || m.k == 0)
                epilogue_rows<T>(part, sx, sz, yo, h * TE, dd, p.has_gate != 0);
            warp_arrive(&bar_part_free[pr]);  // the consumers may reuse this partial slot
            warp_arrive(&bar_sfree[st]);      // x and z of this stage are no longer needed
            fence_proxy_async_smem();         // y rows written by this thread -> visible to the TMA store
            epilogue_sync();
            if (h == 0 && lane == 0 && (!SEQ || p.mode != kModeLocal || m.k == 0)) {  // local pass: segment 0
                const int b = m.b, d0 = m.d0;
                tma_store_3d(&tm_y, smem + S::yout_off + (i % YBUF) * S::yout_bytes, d0, m.t0, b);
                bulk_commit();
                bulk_wait_read<1>();  // the store of the previous tile has read its buffer
            }
            __syncwarp();
        }
        if (h == 0 && lane == 0) bulk_wait_read<0>();
    } else if (warp >= WARP_P0) {
        // ================================================================ P: prologue
        const int h = warp - WARP_P0;
        const T *Bm = static_cast<const T *>(p.Bm);
        const T *Cm = static_cast<const T *>(p.Cm);
        const int c = lane;  // P lane = channel (records)
        float bias_c = 0.f, cb = 0.f;
        float4 cw = make_float4(0.f, 0.f, 0.f, 0.f);
        bool struct_item = false;
        float seg_dsum = 0.f;  // this warp's rows' sum of Delta log2 e over the item
        for (int i = 0;; ++i) {
            const int r = i % R_REC, st = i % STAGES;
            TileMeta *tm = &tmeta[r];
            if (i >= R_REC && !warp_wait(&bar_rec_free[r], uint32_t(i / R_REC - 1) & 1u)) {
                set_timeout(p.status, lane);
                break;
            }
            const bool landed = warp_wait(&bar_full[st], uint32_t(i / STAGES) & 1u);
            TileMeta m = smeta[st];
            if (!landed) {
                set_timeout(p.status, lane);
                m.flags = F_END;
            }
            if (m.flags & F_END) {
                if (h == 0 && lane == 0) *tm = m;
                warp_arrive(&bar_rec_full[r]);
                break;
            }
            const int64_t b = m.b;
            if (m.flags & F_FIRST) {  // new item: channel parameters and the structure of A
                const int64_t d = m.d0 + c;
                const bool ok = d < p.D;
                bias_c = (ok && p.dt_bias) ? __ldg(p.dt_bias + d) : 0.f;
                if (CONV) load_conv(p, d, cw, cb);
                float a[kMaxN];
#pragma unroll
                for (int n = 0; n < kMaxN; ++n) a[n] = (ok && n < p.N) ? __ldg(p.A + d * p.N + n) : 0.f;
                const float dl = (ok && p.N >= 2) ? a[1] - a[0] : 0.f;
                bool arith = true;
#pragma unroll
                for (int n = 2; n < kMaxN; ++n)
                    if (ok && n < p.N && a[n] != a[0] + float(n) * dl) arith = false;
                struct_item = p.allow_structured && __all_sync(0xffffffffu, arith);
            }
            const unsigned char *stage = smem + S::stage_off + size_t(st) * S::stage_bytes;
            float4 *rec = reinterpret_cast<float4 *>(smem + S::rec_off + r * S::rec_bytes) + c;
            float3 x0 = make_float3(0.f, 0.f, 0.f);
            const bool use_x0 = CONV && h == 0 && m.t0 == 0 && conv_prefix<T>(p, m.b, m.d0 + c, x0);
            {
                const T *sx = reinterpret_cast<const T *>(stage + S::st_x) + S::HALO * CH + c;
                T *sdt = reinterpret_cast<T *>(smem + S::stage_off + size_t(st) * S::stage_bytes + S::st_dt) + c;
                // SEQ: the segment's sum of Delta, which the local pass stores
                if (SEQ && (m.flags & F_FIRST)) seg_dsum = 0.f;
                seg_dsum += prologue_rows<T, CONV, TP, SEQ>(sx, sdt, rec, h * TP, m.tlen, bias_c, p.softplus != 0,
                                                            ZOH, cw, cb, use_x0, x0);
                if (SEQ && p.mode == kModeLocal && (m.flags & F_LAST))
                    p.seg_dsum[((m.g * p.K + m.k) * 4 + h) * CH + c] = seg_dsum;
            }
            // u written over dt: order it before the TMA refill of this stage (async proxy)
            if (CONV) fence_proxy_async_smem();
            // B and C rows of this half widened to float32: row t = [B_0 .. B_15 | C_0 .. C_15],
            // in 16-byte chunks; chunk id = q * 32 + lane covers row h*TP + id / 8 and chunk
            // id % 8 (0-3: B, 4-7: C), so eight consecutive lanes write one 128-byte row.
            {
                float *bcf = reinterpret_cast<float *>(smem + S::bcf_off + r * S::bcf_bytes);
#pragma unroll
                for (int q = 0; q < TP * 8 / 32; ++q) {
                    const int id = q * 32 + lane, t = h * TP + (id >> 3), j = id & 7;
                    const int n0 = (j & 3) * 4;
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (t < m.tlen) {
                        if (p.bc_tma) {
                            v = Tok<T>::quad(reinterpret_cast<const T *>(stage + (j < 4 ? S::st_b : S::st_c)) +
                                             t * kMaxN + n0);
                        } else {
                            const T *src = (j < 4 ? Bm : Cm) + (b * p.L + m.t0 + t) * p.N + n0;
                            v.x = n0 < p.N ? Tok<T>::ldg(src) : 0.f;
                            v.y = n0 + 1 < p.N ? Tok<T>::ldg(src + 1) : 0.f;
                            v.z = n0 + 2 < p.N ? Tok<T>::ldg(src + 2) : 0.f;
                            v.w = n0 + 3 < p.N ? Tok<T>::ldg(src + 3) : 0.f;
                        }
                    }
                    *reinterpret_cast<float4 *>(bcf + t * 32 + j * 4) = v;
                }
            }
            if (h == 0 && lane == 0) {
                TileMeta mm = m;
                mm.flags |= struct_item ? F_STRUCT : 0;
                *tm = mm;
            }
            warp_arrive(&bar_rec_full[r]);
            warp_arrive(&bar_sfree[st]);  // x, dt, B, C of this stage read (E still reads x, z)
        }
    } else {
        // ============================================================ consumers
        const int c = lane;  // channel within the group
        const int w = warp;  // states 4w .. 4w+3
        float2 h01 = f2(0.f, 0.f), h23 = f2(0.f, 0.f);
        float4 Aq = make_float4(0.f, 0.f, 0.f, 0.f), zA = Aq, iA = Aq;
        float del = 0.f;
        for (int i = 0;; ++i) {
            const int r = i % R_REC, pr = i % R_PART;
            const bool have = warp_wait(&bar_rec_full[r], uint32_t(i / R_REC) & 1u);
            const TileMeta m = tmeta[r];
            if (!have || (m.flags & F_END)) {
                if (!have) set_timeout(p.status, lane);
                // E reads the end marker from its stage. Arrive only once E has released the
                // slot's previous use: a phase-parity wait cannot tell phase u from u + 2.
                if (i < R_PART || warp_wait(&bar_part_free[pr], uint32_t(i / R_PART - 1) & 1u))
                    warp_arrive(&bar_part_full[pr]);
                break;
            }
            const int64_t b = m.b;
            const int64_t d = m.d0 + c;
            const bool dvalid = d < p.D;
            if (m.flags & F_FIRST) {
                float a[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int n = 4 * w + j;
                    a[j] = (dvalid && n < p.N) ? __ldg(p.A + d * p.N + n) : 0.f;
                }
                Aq = make_float4(a[0], a[1], a[2], a[3]);
                if (ZOH) {
                    zA = make_float4(a[0] * kLn2, a[1] * kLn2, a[2] * kLn2, a[3] * kLn2);
                    iA = make_float4(a[0] != 0.f ? 1.f / a[0] : 0.f, a[1] != 0.f ? 1.f / a[1] : 0.f,
                                     a[2] != 0.f ? 1.f / a[2] : 0.f, a[3] != 0.f ? 1.f / a[3] : 0.f);
                }
                del = (dvalid && p.N >= 2) ? __ldg(p.A + d * p.N + 1) - __ldg(p.A + d * p.N) : 0.f;
                if (SEQ && m.k > 0 && p.mode == kModeLocal) {  // the local pass: every later segment from zero
                    h01 = f2(0.f, 0.f);
                    h23 = f2(0.f, 0.f);
                } else if (SEQ && m.k > 0 && p.mode == kModeFromCarry) {  // the combine kernel's start state
                    const float4 hv =
                        __ldcg(reinterpret_cast<const float4 *>(p.seg_state) + ((m.g * p.K + m.k) * CW + w) * CH + c);
                    h01 = f2(hv.x, hv.y);
                    h23 = f2(hv.z, hv.w);
                } else if (m.k == 0) {
                    float hv[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int n = 4 * w + j;
                        hv[j] = (dvalid && n < p.N && p.h0) ? __ldg(p.h0 + (b * p.D + d) * p.N + n) : 0.f;
                    }
                    h01 = f2(hv[0], hv[1]);
                    h23 = f2(hv[2], hv[3]);
                } else {
                    // The predecessor segment (g, k-1) was claimed earlier by a running block.
                    if (lane == 0 && ld_acquire_gpu(p.flags + m.g) < uint32_t(m.k)) {
                        const uint64_t start = globaltimer_ns();
                        for (uint32_t it = 1;; ++it) {
                            if (ld_acquire_gpu(p.flags + m.g) >= uint32_t(m.k)) break;
                            __nanosleep(128);
                            if ((it & 63u) == 0 && globaltimer_ns() - start > kWaitLimitNs) {
                                atomicExch(p.status, uint32_t(SSM_ERR_TIMEOUT));
                                break;  // carry on with what is there; the status reports it
                            }
                        }
                    }
                    __syncwarp();
                    __threadfence();
                    const float4 hv = __ldcg(reinterpret_cast<const float4 *>(p.carry) + (m.g * CW + w) * CH + c);
                    h01 = f2(hv.x, hv.y);
                    h23 = f2(hv.z, hv.w);
                }
            }
            if (i >= R_PART && !warp_wait(&bar_part_free[pr], uint32_t(i / R_PART - 1) & 1u)) {
                set_timeout(p.status, lane);
                break;
            }
            const float4 *rec = reinterpret_cast<const float4 *>(smem + S::rec_off + r * S::rec_bytes) + c;
            const float *bc = reinterpret_cast<const float *>(smem + S::bcf_off + r * S::bcf_bytes) + 4 * w;
            float4 *part = reinterpret_cast<float4 *>(smem + S::part_off + pr * S::part_bytes) + w * (TT / 4) * CH + c;
            // With one block per SM the registers allow the factors to run a block ahead.
            constexpr bool kAhead = C::MINB == 1;
            if (m.flags & F_STRUCT) consume_tile<true, ZOH, kAhead>(rec, bc, part, Aq, del, zA, iA, h01, h23);
            else consume_tile<false, ZOH, kAhead>(rec, bc, part, Aq, del, zA, iA, h01, h23);
            warp_arrive(&bar_rec_free[r]);
            warp_arrive(&bar_part_full[pr]);
            if (SEQ && (m.flags & F_LAST) && p.mode == kModeLocal) {
                reinterpret_cast<float4 *>(p.seg_local)[((m.g * p.K + m.k) * CW + w) * CH + c] =
                    make_float4(h01.x, h01.y, h23.x, h23.y);
            } else if (SEQ && (m.flags & F_LAST) && p.mode == kModeFromCarry) {
                if (m.k == p.K - 1 && p.h_last && dvalid) {
                    const float hv[4] = {h01.x, h01.y, h23.x, h23.y};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int n = 4 * w + j;
                        if (n < p.N) p.h_last[(b * p.D + d) * p.N + n] = hv[j];
                    }
                }
            } else if (m.flags & F_LAST) {
                if (m.k == p.K - 1) {
                    if (p.h_last && dvalid) {
                        const float hv[4] = {h01.x, h01.y, h23.x, h23.y};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int n = 4 * w + j;
                            if (n < p.N) p.h_last[(b * p.D + d) * p.N + n] = hv[j];
                        }
                    }
                } else {
                    reinterpret_cast<float4 *>(p.carry)[(m.g * CW + w) * CH + c] = make_float4(h01.x, h01.y, h23.x, h23.y);
                    consumer_sync();
                    if (threadIdx.x == 0 && !(p.drop_handoff && m.g == 0 && m.k == 0)) {
                        __threadfence();
                        st_release_gpu(p.flags + m.g, uint32_t(m.k + 1));
                    }
                }
            }
        }
    }
}

}  // namespace scan
}  // namespace ssm
