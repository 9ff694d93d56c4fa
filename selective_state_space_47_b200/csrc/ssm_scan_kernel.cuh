// ssm_scan_kernel.cuh -- warp-specialised selective-scan forward kernel for sm_100a.
//
// One thread block owns one group of CH = 32 channels of one sequence at a time
// and walks the item's time segment tile by tile (TT steps per tile). Six warps
// with fixed roles, connected by mbarrier rings (every wait bounded in time and
// suspended in hardware while it waits):
//
//   W0..W3  consumers    the recurrence. Lane c is channel c of the group; warp w
//                        keeps states 4w .. 4w+3 of its lane's channel in registers.
//                        Per step a lane reads its channel's 8-byte record (u, Delta
//                        log2 e) and, with one warp-uniform broadcast load each, the
//                        B_t and C_t values of the warp's four states; it forms Abar,
//                        updates h = Abar h + u B and its partial readout sum_n C_n h_n
//                        (one 16-byte store per four steps).
//   P       prologue     per (t, channel), once: Delta = softplus(dt + bias), u = Delta
//                        x, Delta log2 e; widens the B and C rows to float32.
//   E       epilogue     per (t, channel): sums the four warps' partials, adds D x,
//                        applies the SiLU gate, rounds, stores the y tile with TMA; it
//                        also claims the (group, segment) items and issues the TMA
//                        loads of x, dt, z, B, C into a STAGES-deep ring (it is the last
//                        reader of a stage, so it refills it).
//
// Why this shape: shared memory delivers 128 bytes per clock per SM to registers,
// and a 16-byte load whose 32 lanes read different addresses costs four of those
// clocks, while one whose lanes all read the same address costs one. With lanes
// over channels and warps over states, B_t and C_t (shared by all channels) are
// warp-uniform, and the only lane-distinct data per step is the 8-byte record.
//
// Rings: stage (TMA, STAGES deep) -> P -> record ring (R_REC deep) -> consumers ->
// partial ring (R_PART deep) -> E. Between blocks, an item (group g, segment k)
// starts from the state its predecessor (g, k-1) published in the workspace.
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
constexpr int CH = 32;                            // channels per block (one per lane)
constexpr int NTHREADS = (CW + 2) * 32;           // consumers + P + E
constexpr int WARP_P = CW, WARP_E = CW + 1;
constexpr int TT = 32;                            // time steps per tile
#ifndef SSM_STAGES
#define SSM_STAGES 4
#endif
constexpr int STAGES = SSM_STAGES;                // TMA ring depth (tiles)
constexpr int R_REC = 3;                          // record ring depth
constexpr int R_PART = 2;                         // partial-sum ring depth
constexpr int kMaxN = 16;                         // state slots per channel
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // every device-side wait gives up after 2 s
constexpr uint32_t kSuspendNs = 20000;            // hardware suspend hint per try_wait

enum : int { F_FIRST = 1, F_LAST = 2, F_END = 4, F_STRUCT = 8 };

struct TileMeta {
    long long g, k;  // channel group and time segment of the tile's item
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
    int has_gate, softplus, allow_structured, drop_handoff, bc_tma;
};

template <typename T>
struct Layout {
    static constexpr int BOX = TT * CH;           // elements of one token box [TT][CH]
    static constexpr int BCBOX = TT * kMaxN;      // elements of one B or C box [TT][16]
    static constexpr size_t tok_bytes = size_t(BOX) * sizeof(T);
    static constexpr size_t bc_bytes = size_t(BCBOX) * sizeof(T);
    static constexpr size_t stage_bytes = 3 * tok_bytes + 2 * bc_bytes;
    static constexpr size_t stage_off = 0;
    static constexpr size_t rec_off = stage_off + STAGES * stage_bytes;
    static constexpr size_t rec_bytes = size_t(BOX) * 8;            // float2 (u, Delta log2 e) per (t, c)
    static constexpr size_t bcf_off = rec_off + R_REC * rec_bytes;
    static constexpr size_t bcf_bytes = size_t(TT) * 32 * 4;        // [TT][B 16 | C 16] float
    static constexpr size_t part_off = bcf_off + R_REC * bcf_bytes;
    static constexpr size_t part_bytes = size_t(CW) * (TT / 4) * CH * 16;  // [w][t/4][c] float4
    static constexpr size_t yout_off = part_off + R_PART * part_bytes;
    static constexpr size_t yout_bytes = tok_bytes;
    static constexpr size_t dsk_off = yout_off + 2 * yout_bytes;
    static constexpr size_t smeta_off = dsk_off + STAGES * CH * 4;
    static constexpr size_t tmeta_off = smeta_off + STAGES * sizeof(TileMeta);
    static constexpr size_t bar_off = (tmeta_off + R_REC * sizeof(TileMeta) + 15) / 16 * 16;
    static constexpr int NBARS = STAGES + 2 * R_REC + 2 * R_PART;
    static constexpr size_t total = bar_off + NBARS * 8;
    static_assert(stage_bytes % 128 == 0 && tok_bytes % 128 == 0, "TMA boxes must stay 128-byte aligned");
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

__device__ __forceinline__ void consumer_sync() {  // named barrier 1: the consumer warps only
    asm volatile("bar.sync 1, %0;" ::"n"(CW * 32) : "memory");
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// softplus of two values: log(1 + e^v), series for e^v < 2^-6, v itself above 15.
__device__ __forceinline__ float2 softplus2(float2 v) {
    const float2 x = __fmul2_rn(v, f2(kLog2e, kLog2e));
    const float2 e = f2(ex2_approx(x.x), ex2_approx(x.y));
    float2 s = __ffma2_rn(e, f2(-0.25f, -0.25f), f2(0.33333334f, 0.33333334f));
    s = __ffma2_rn(e, s, f2(-0.5f, -0.5f));
    s = __ffma2_rn(e, s, f2(1.f, 1.f));
    s = __fmul2_rn(e, s);
    const float2 one_e = __fadd2_rn(e, f2(1.f, 1.f));
    const float2 lg = __fmul2_rn(f2(lg2_approx(one_e.x), lg2_approx(one_e.y)), f2(kLn2, kLn2));
    float2 r;
    r.x = v.x > 15.f ? v.x : (e.x < 0.015625f ? s.x : lg.x);
    r.y = v.y > 15.f ? v.y : (e.y < 0.015625f ? s.y : lg.y);
    return r;
}

// silu of two values: z / (1 + e^-z).
__device__ __forceinline__ float2 silu2(float2 z) {
    const float2 nz = __fmul2_rn(z, f2(-kLog2e, -kLog2e));
    const float2 den = __fadd2_rn(f2(ex2_approx(nz.x), ex2_approx(nz.y)), f2(1.f, 1.f));
    return __fmul2_rn(z, f2(rcp_approx(den.x), rcp_approx(den.y)));
}

// ---------------------------------------------------------------- consumers
// TT steps of one tile for one lane (its channel, the warp's four states).
// rec: this lane's records (stride CH float2 per step); bc: B of the warp's states
// (stride 32 floats per step; C at +16); part: this lane's partials (stride CH
// float4 per block of four steps). Aq: A[c][4w .. 4w+3]; del: A[c][1] - A[c][0].
template <bool STRUCT>
__device__ __forceinline__ void consume_tile(const float2 *__restrict__ rec, const float *__restrict__ bc,
                                             float4 *__restrict__ part, const float4 Aq, const float del,
                                             float2 &h01, float2 &h23) {
#pragma unroll
    for (int t4 = 0; t4 < TT; t4 += 4) {
        float yv[4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int t = t4 + s;
            const float2 p = rec[t * CH];  // (u, Delta log2 e)
            const float4 b4 = *reinterpret_cast<const float4 *>(bc + t * 32);       // warp-uniform
            const float4 c4 = *reinterpret_cast<const float4 *>(bc + t * 32 + 16);  // warp-uniform
            float2 a01, a23;
            if (STRUCT) {
                const float2 x = __fmul2_rn(f2(p.y, p.y), f2(Aq.x, del));
                const float a0 = ex2_approx(x.x), r = ex2_approx(x.y);
                a01 = f2(a0, a0 * r);
                a23 = __fmul2_rn(a01, f2(r * r, r * r));
            } else {
                const float2 x01 = __fmul2_rn(f2(p.y, p.y), f2(Aq.x, Aq.y));
                const float2 x23 = __fmul2_rn(f2(p.y, p.y), f2(Aq.z, Aq.w));
                a01 = f2(ex2_approx(x01.x), ex2_approx(x01.y));
                a23 = f2(ex2_approx(x23.x), ex2_approx(x23.y));
            }
            const float2 u2 = f2(p.x, p.x);
            h01 = __ffma2_rn(a01, h01, __fmul2_rn(u2, f2(b4.x, b4.y)));
            h23 = __ffma2_rn(a23, h23, __fmul2_rn(u2, f2(b4.z, b4.w)));
            const float2 yy = __ffma2_rn(f2(c4.z, c4.w), h23, __fmul2_rn(f2(c4.x, c4.y), h01));
            yv[s] = yy.x + yy.y;
        }
        part[(t4 / 4) * CH] = make_float4(yv[0], yv[1], yv[2], yv[3]);
    }
}

// ------------------------------------------------------------------- kernel
template <typename T>
__global__ void __launch_bounds__(NTHREADS)
    scan_ws_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_dt,
                   const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                   const Params p) {
    using S = Layout<T>;
    extern __shared__ __align__(1024) unsigned char smem[];
    TileMeta *smeta = reinterpret_cast<TileMeta *>(smem + S::smeta_off);  // per TMA stage
    TileMeta *tmeta = reinterpret_cast<TileMeta *>(smem + S::tmeta_off);  // per record slot
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(smem + S::bar_off);
    uint64_t *bar_rec_full = bar_tma + STAGES;
    uint64_t *bar_rec_free = bar_rec_full + R_REC;
    uint64_t *bar_part_full = bar_rec_free + R_REC;
    uint64_t *bar_part_free = bar_part_full + R_PART;
    float *dsk = reinterpret_cast<float *>(smem + S::dsk_off);  // D of the tile's channels, per stage
    auto stage_ptr = [&](int s) { return smem + S::stage_off + size_t(s) * S::stage_bytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(&bar_tma[s], 1);
        for (int r = 0; r < R_REC; ++r) {
            mbar_init(&bar_rec_full[r], 32);
            mbar_init(&bar_rec_free[r], CW * 32);
        }
        for (int r = 0; r < R_PART; ++r) {
            mbar_init(&bar_part_full[r], CW * 32);
            mbar_init(&bar_part_free[r], 32);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == WARP_E) {
        // ====================================================== E: epilogue + loads
        const int ntok = p.has_gate ? 3 : 2;
        const uint32_t tx_bytes = uint32_t(ntok * S::tok_bytes + (p.bc_tma ? 2 * S::bc_bytes : 0));
        if (lane == 0) {
            prefetch_tensormap(&tm_x);
            prefetch_tensormap(&tm_dt);
            if (p.has_gate) prefetch_tensormap(&tm_z);
            if (p.bc_tma) {
                prefetch_tensormap(&tm_b);
                prefetch_tensormap(&tm_c);
            }
            prefetch_tensormap(&tm_y);
        }
        long long li_g = 0, li_k = 0, li_beg = 0, li_end = 0;
        int li_j = 0, li_n = 0;
        bool li_ok = false;
        auto claim = [&]() {
            unsigned int it = 0;
            if (lane == 0) it = atomicAdd(p.counter, 1u);
            it = __shfl_sync(0xffffffffu, it, 0);
            li_ok = (long long)it < p.items;
            if (li_ok) {
                li_k = (long long)it / p.G;
                li_g = (long long)it % p.G;
                li_beg = li_k * p.seg_len;
                li_end = min((long long)p.L, li_beg + p.seg_len);
                li_n = int((li_end - li_beg + TT - 1) / TT);
                li_j = 0;
            }
        };
        auto issue = [&](int st) {  // fetch the next tile of the stream into stage st
            TileMeta m;
            m.g = li_g;
            m.k = li_k;
            m.j = li_j;
            m.t0 = int(li_beg + (long long)li_j * TT);
            m.tlen = int(li_end - m.t0 < TT ? li_end - m.t0 : TT);
            m.flags = li_ok ? ((li_j == 0 ? F_FIRST : 0) | (li_j == li_n - 1 ? F_LAST : 0)) : F_END;
            if (lane == 0) {
                smeta[st] = m;
                if (li_ok) {
                    unsigned char *stage = stage_ptr(st);
                    const int b = int(m.g / p.Dg), d0 = int((m.g % p.Dg) * CH);
                    mbar_arrive_expect_tx(&bar_tma[st], tx_bytes);
                    tma_load_3d(stage, &tm_x, &bar_tma[st], d0, m.t0, b);
                    tma_load_3d(stage + S::tok_bytes, &tm_dt, &bar_tma[st], d0, m.t0, b);
                    if (p.has_gate) tma_load_3d(stage + 2 * S::tok_bytes, &tm_z, &bar_tma[st], d0, m.t0, b);
                    if (p.bc_tma) {
                        tma_load_3d(stage + 3 * S::tok_bytes, &tm_b, &bar_tma[st], 0, m.t0, b);
                        tma_load_3d(stage + 3 * S::tok_bytes + S::bc_bytes, &tm_c, &bar_tma[st], 0, m.t0, b);
                    }
                } else {
                    mbar_arrive(&bar_tma[st]);  // end of the stream: complete the phase without data
                }
            }
            __syncwarp();
            if (li_ok && ++li_j == li_n) claim();
        };

        claim();
        for (int s = 0; s < STAGES; ++s) issue(s);

        const int c = lane;  // E lane = channel
        for (int i = 0;; ++i) {
            const int pr = i % R_PART, st = i % STAGES;
            if (!warp_wait(&bar_part_full[pr], uint32_t(i / R_PART) & 1u)) {
                if (lane == 0) atomicExch(p.status, uint32_t(SSM_ERR_TIMEOUT));
                break;
            }
            const TileMeta m = smeta[st];
            if (m.flags & F_END) break;
            const unsigned char *stage = stage_ptr(st);
            const T *sx = reinterpret_cast<const T *>(stage);
            const T *sz = reinterpret_cast<const T *>(stage + 2 * S::tok_bytes);
            const float4 *part = reinterpret_cast<const float4 *>(smem + S::part_off + pr * S::part_bytes);
            T *yo = reinterpret_cast<T *>(smem + S::yout_off + (i & 1) * S::yout_bytes);
            const float dd = dsk[st * CH + c];
#pragma unroll 2
            for (int blk = 0; blk < TT / 4; ++blk) {
                float4 acc = part[(0 * (TT / 4) + blk) * CH + c];
#pragma unroll
                for (int w = 1; w < CW; ++w) {
                    const float4 v = part[(w * (TT / 4) + blk) * CH + c];
                    const float2 lo = __fadd2_rn(f2(acc.x, acc.y), f2(v.x, v.y));
                    const float2 hi = __fadd2_rn(f2(acc.z, acc.w), f2(v.z, v.w));
                    acc = make_float4(lo.x, lo.y, hi.x, hi.y);
                }
                const int t = blk * 4;
                const float2 x01 = f2(Tok<T>::to_f(sx[t * CH + c]), Tok<T>::to_f(sx[(t + 1) * CH + c]));
                const float2 x23 = f2(Tok<T>::to_f(sx[(t + 2) * CH + c]), Tok<T>::to_f(sx[(t + 3) * CH + c]));
                float2 y01 = __ffma2_rn(f2(dd, dd), x01, f2(acc.x, acc.y));
                float2 y23 = __ffma2_rn(f2(dd, dd), x23, f2(acc.z, acc.w));
                if (p.has_gate) {
                    const float2 z01 = f2(Tok<T>::to_f(sz[t * CH + c]), Tok<T>::to_f(sz[(t + 1) * CH + c]));
                    const float2 z23 = f2(Tok<T>::to_f(sz[(t + 2) * CH + c]), Tok<T>::to_f(sz[(t + 3) * CH + c]));
                    y01 = __fmul2_rn(y01, silu2(z01));
                    y23 = __fmul2_rn(y23, silu2(z23));
                }
                yo[t * CH + c] = Tok<T>::from_f(y01.x);
                yo[(t + 1) * CH + c] = Tok<T>::from_f(y01.y);
                yo[(t + 2) * CH + c] = Tok<T>::from_f(y23.x);
                yo[(t + 3) * CH + c] = Tok<T>::from_f(y23.y);
            }
            mbar_arrive(&bar_part_free[pr]);  // the consumers may reuse this partial slot
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int b = int(m.g / p.Dg), d0 = int((m.g % p.Dg) * CH);
                tma_store_3d(&tm_y, yo, d0, m.t0, b);
                bulk_commit();
                bulk_wait_read<1>();  // the store issued from the other y buffer has read it
            }
            __syncwarp();
            issue(st);  // stage st is no longer needed: refill it with the next tile of the stream
        }
        if (lane == 0) bulk_wait_read<0>();
    } else if (warp == WARP_P) {
        // ============================================================ P: prologue
        const T *Bm = static_cast<const T *>(p.Bm);
        const T *Cm = static_cast<const T *>(p.Cm);
        const int c = lane;  // P lane = channel
        float bias_c = 0.f, dsk_c = 0.f;
        bool struct_item = false;
        for (int i = 0;; ++i) {
            const int r = i % R_REC, st = i % STAGES;
            TileMeta *tm = &tmeta[r];
            if (i >= R_REC && !warp_wait(&bar_rec_free[r], uint32_t(i / R_REC - 1) & 1u)) {
                if (lane == 0) atomicExch(p.status, uint32_t(SSM_ERR_TIMEOUT));
                break;
            }
            const bool landed = warp_wait(&bar_tma[st], uint32_t(i / STAGES) & 1u);
            TileMeta m = smeta[st];
            if (!landed) {
                if (lane == 0) atomicExch(p.status, uint32_t(SSM_ERR_TIMEOUT));
                m.flags = F_END;
            }
            if (m.flags & F_END) {
                if (lane == 0) *tm = m;
                __syncwarp();
                mbar_arrive(&bar_rec_full[r]);
                break;
            }
            const int64_t b = m.g / p.Dg;
            const int64_t d = (m.g % p.Dg) * CH + c;
            if (m.flags & F_FIRST) {  // new item: channel parameters and the structure of A
                const bool ok = d < p.D;
                bias_c = (ok && p.dt_bias) ? __ldg(p.dt_bias + d) : 0.f;
                dsk_c = (ok && p.Dskip) ? __ldg(p.Dskip + d) : 0.f;
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
            // Records: one per (t, channel), two steps at a time.
            const unsigned char *stage = stage_ptr(st);
            const T *sx = reinterpret_cast<const T *>(stage);
            const T *sdt = reinterpret_cast<const T *>(stage + S::tok_bytes);
            float2 *rec = reinterpret_cast<float2 *>(smem + S::rec_off + r * S::rec_bytes);
#pragma unroll 4
            for (int t = 0; t < TT; t += 2) {
                const float2 v = __fadd2_rn(f2(Tok<T>::to_f(sdt[t * CH + c]), Tok<T>::to_f(sdt[(t + 1) * CH + c])),
                                            f2(bias_c, bias_c));
                const float2 delta = p.softplus ? softplus2(v) : v;
                const float2 dlg = __fmul2_rn(delta, f2(kLog2e, kLog2e));
                const float2 u = __fmul2_rn(delta, f2(Tok<T>::to_f(sx[t * CH + c]), Tok<T>::to_f(sx[(t + 1) * CH + c])));
                // Past the end of the sequence: u = 0 and Delta = 0 give Abar = 1 and no input.
                rec[t * CH + c] = t < m.tlen ? f2(u.x, dlg.x) : f2(0.f, 0.f);
                rec[(t + 1) * CH + c] = t + 1 < m.tlen ? f2(u.y, dlg.y) : f2(0.f, 0.f);
            }
            // B and C rows widened to float32: row t = [B_0 .. B_15 | C_0 .. C_15]; id =
            // mq * 32 + lane covers row id / 8 and quarter id % 8 (quarters 0-3 B, 4-7 C).
            float *bcf = reinterpret_cast<float *>(smem + S::bcf_off + r * S::bcf_bytes);
#pragma unroll
            for (int mq = 0; mq < TT * 8 / 32; ++mq) {
                const int id = mq * 32 + lane, t = id >> 3, k = id & 7;
                const int n0 = (k & 3) * 4;
                float v[4];
                if (t >= m.tlen) {
                    v[0] = v[1] = v[2] = v[3] = 0.f;
                } else if (p.bc_tma) {
                    const T *src = reinterpret_cast<const T *>(stage + 3 * S::tok_bytes + (k < 4 ? 0 : S::bc_bytes));
#pragma unroll
                    for (int e = 0; e < 4; ++e) v[e] = Tok<T>::to_f(src[t * kMaxN + n0 + e]);
                } else {
                    const T *src = k < 4 ? Bm : Cm;
                    const int64_t tt = m.t0 + t;
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        v[e] = (n0 + e < p.N) ? Tok<T>::ldg(src + (b * p.L + tt) * p.N + n0 + e) : 0.f;
                }
                *reinterpret_cast<float4 *>(bcf + t * 32 + k * 4) = make_float4(v[0], v[1], v[2], v[3]);
            }
            dsk[st * CH + c] = dsk_c;
            if (lane == 0) {
                TileMeta mm = m;
                mm.flags |= struct_item ? F_STRUCT : 0;
                *tm = mm;
            }
            __syncwarp();
            mbar_arrive(&bar_rec_full[r]);
        }
    } else {
        // ============================================================ consumers
        const int c = lane;  // channel within the group
        const int w = warp;  // states 4w .. 4w+3
        float2 h01 = f2(0.f, 0.f), h23 = f2(0.f, 0.f);
        float4 Aq = make_float4(0.f, 0.f, 0.f, 0.f);
        float del = 0.f;
        for (int i = 0;; ++i) {
            const int r = i % R_REC, pr = i % R_PART;
            const bool have = warp_wait(&bar_rec_full[r], uint32_t(i / R_REC) & 1u);
            const TileMeta m = tmeta[r];
            if (!have || (m.flags & F_END)) {
                if (!have && lane == 0) atomicExch(p.status, uint32_t(SSM_ERR_TIMEOUT));
                // E reads the end marker from its stage. Arrive only once E has released the
                // slot's previous use: a phase-parity wait cannot tell phase u from u + 2.
                if (i < R_PART || warp_wait(&bar_part_free[pr], uint32_t(i / R_PART - 1) & 1u))
                    mbar_arrive(&bar_part_full[pr]);
                break;
            }
            const int64_t b = m.g / p.Dg;
            const int64_t d = (m.g % p.Dg) * CH + c;
            const bool dvalid = d < p.D;
            if (m.flags & F_FIRST) {
                float a[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int n = 4 * w + j;
                    a[j] = (dvalid && n < p.N) ? __ldg(p.A + d * p.N + n) : 0.f;
                }
                Aq = make_float4(a[0], a[1], a[2], a[3]);
                del = (dvalid && p.N >= 2) ? __ldg(p.A + d * p.N + 1) - __ldg(p.A + d * p.N) : 0.f;
                if (m.k == 0) {
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
                if (lane == 0) atomicExch(p.status, uint32_t(SSM_ERR_TIMEOUT));
                break;
            }
            const float2 *rec = reinterpret_cast<const float2 *>(smem + S::rec_off + r * S::rec_bytes) + c;
            const float *bc = reinterpret_cast<const float *>(smem + S::bcf_off + r * S::bcf_bytes) + 4 * w;
            float4 *part = reinterpret_cast<float4 *>(smem + S::part_off + pr * S::part_bytes) + w * (TT / 4) * CH + c;
            if (m.flags & F_STRUCT) consume_tile<true>(rec, bc, part, Aq, del, h01, h23);
            else consume_tile<false>(rec, bc, part, Aq, del, h01, h23);
            mbar_arrive(&bar_rec_free[r]);
            mbar_arrive(&bar_part_full[pr]);
            if (m.flags & F_LAST) {
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
