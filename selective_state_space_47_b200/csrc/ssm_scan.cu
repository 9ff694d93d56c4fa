// ssm_scan.cu -- B200 (sm_100a) kernels and C ABI of the selective state space
// (S6) forward scan and the recurrent one-token step.
//
// Scan kernel layout (one thread block = one group of CH channels of one
// sequence, CH = 8 * warps):
//   * four lanes per channel, each lane owning four of the N <= 16 states
//     (states q, q+4, q+8, q+12 for lane q of the channel); the state stays in
//     registers for the whole time segment;
//   * tokens x, dt, z arrive as [TT x CH] boxes through a 3-stage TMA ring;
//     B_t and C_t rows are prefetched into registers one tile ahead;
//   * a per-tile prologue computes, once per (t, channel), Delta = softplus(dt +
//     bias), u = Delta x and the exponent scale; the main loop then does the
//     state update and the per-lane partial readout, and every four steps the
//     four lanes of a channel reduce-scatter their partial sums so that each
//     lane finalises one token (D skip, SiLU gate, store);
//   * y leaves through a TMA store of each [TT x CH] tile.
// Sequence parallelism: the sequence of a channel group is cut into time
// segments; (group, segment) items are handed out in order by an atomic
// counter, and an item starts from the state its predecessor publishes in the
// workspace (bounded wait on a release/acquire flag). The recurrence is
// associative (Mamba summary, azimuth.plus, hardware-aware algorithm
// paragraph: parallel scan), so the segmented evaluation is exact and every
// exponential is computed once.
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "../../include/ssm_scan.h"
#include "ssm_device.cuh"

using namespace ssm;

namespace {

constexpr int TT = 32;      // time steps per tile
constexpr int STAGES = 3;   // depth of the TMA input ring
constexpr int kMaxN = 16;   // states per channel handled by the kernels
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bound on every device-side wait (2 s)

// ------------------------------------------------------------- workspace
// [0, 4) item counter; [4, 8) device status; [256, ...) per-group flags;
// then per-group hand-off states float32 [G][CH][16].
constexpr size_t kWsHeader = 256;

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct ScanParams {
    int64_t L, D, N;
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
    int has_gate, softplus, allow_structured, drop_handoff;
};

template <typename T, int WARPS>
struct ScanSmem {
    static constexpr int CH = 8 * WARPS;
    static constexpr int BOX = TT * CH;
    static constexpr size_t in_off = 0;
    static constexpr size_t in_bytes = size_t(STAGES) * 3 * BOX * sizeof(T);
    static constexpr size_t y_off = in_off + in_bytes;
    static constexpr size_t y_bytes = size_t(2) * BOX * sizeof(T);
    static constexpr size_t pro_off = y_off + y_bytes;
    static constexpr size_t pro_bytes = size_t(BOX) * 16;
    static constexpr size_t bc_off = pro_off + pro_bytes;
    static constexpr size_t bc_bytes = size_t(TT) * 32 * 4;
    static constexpr size_t par_off = bc_off + bc_bytes;
    static constexpr size_t par_bytes = size_t(2) * CH * 4;
    static constexpr size_t bar_off = (par_off + par_bytes + 15) / 16 * 16;
    static constexpr size_t item_off = bar_off + STAGES * 8;
    static constexpr size_t total = item_off + 8;
};

// Wait for the phase `parity` of an mbarrier, bounded in time. Returns false on timeout.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0 && globaltimer_ns() - start > kWaitLimitNs) return false;
    }
}

// One tile of the time loop for one lane: TT steps of the recurrence for the
// lane's four states, with the four-lane reduce-scatter of the readout every
// four steps and the epilogue of the token this lane finalises.
template <typename T, int CH, bool STRUCT, bool GATE>
__device__ __forceinline__ void scan_tile(const float4 *__restrict__ s_pro, const float *__restrict__ s_bc,
                                          const T *__restrict__ sx, const T *__restrict__ sz,
                                          T *__restrict__ sy, const int cl, const int q, const float (&Al)[4],
                                          const float Dd, float (&h)[4]) {
    constexpr unsigned FULL = 0xffffffffu;
    const bool hi2 = (q & 2) != 0, hi1 = (q & 1) != 0;
#pragma unroll 2
    for (int t4 = 0; t4 < TT; t4 += 4) {
        float yp[4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int t = t4 + s;
            const float4 pr = s_pro[t * CH + cl];  // (u = Delta x, Delta log2e, ratio for n -> n+4, -)
            const float4 bq = *reinterpret_cast<const float4 *>(s_bc + t * 32 + q * 4);
            const float4 cq = *reinterpret_cast<const float4 *>(s_bc + t * 32 + 16 + q * 4);
            float a0, a1, a2, a3;
            if (STRUCT) {
                a0 = ex2_approx(pr.y * Al[0]);
                a1 = a0 * pr.z;
                a2 = a1 * pr.z;
                a3 = a2 * pr.z;
            } else {
                a0 = ex2_approx(pr.y * Al[0]);
                a1 = ex2_approx(pr.y * Al[1]);
                a2 = ex2_approx(pr.y * Al[2]);
                a3 = ex2_approx(pr.y * Al[3]);
            }
            h[0] = fmaf(a0, h[0], pr.x * bq.x);
            h[1] = fmaf(a1, h[1], pr.x * bq.y);
            h[2] = fmaf(a2, h[2], pr.x * bq.z);
            h[3] = fmaf(a3, h[3], pr.x * bq.w);
            yp[s] = fmaf(cq.x, h[0], fmaf(cq.y, h[1], fmaf(cq.z, h[2], cq.w * h[3])));
        }
        // Reduce-scatter over the channel's four lanes: lane q ends with the
        // full readout of step t4 + q.
        const float send0 = hi2 ? yp[0] : yp[2], send1 = hi2 ? yp[1] : yp[3];
        float keep0 = hi2 ? yp[2] : yp[0], keep1 = hi2 ? yp[3] : yp[1];
        keep0 += __shfl_xor_sync(FULL, send0, 2);
        keep1 += __shfl_xor_sync(FULL, send1, 2);
        const float send2 = hi1 ? keep0 : keep1;
        float yv = hi1 ? keep1 : keep0;
        yv += __shfl_xor_sync(FULL, send2, 1);
        const int e = (t4 + q) * CH + cl;
        yv = fmaf(Dd, Tok<T>::to_f(sx[e]), yv);
        if (GATE) yv *= silu_f(Tok<T>::to_f(sz[e]));
        sy[e] = Tok<T>::from_f(yv);
    }
}

template <typename T, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
    scan_fwd_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_dt,
                    const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_y,
                    const ScanParams p) {
    using S = ScanSmem<T, WARPS>;
    constexpr int CH = S::CH, BOX = S::BOX, NT = WARPS * 32;
    constexpr int BC_PER_THREAD = TT * 32 / NT;
    extern __shared__ __align__(1024) unsigned char smem[];
    T *s_in = reinterpret_cast<T *>(smem + S::in_off);
    T *s_y = reinterpret_cast<T *>(smem + S::y_off);
    float4 *s_pro = reinterpret_cast<float4 *>(smem + S::pro_off);
    float *s_bc = reinterpret_cast<float *>(smem + S::bc_off);
    float *s_bias = reinterpret_cast<float *>(smem + S::par_off);
    float *s_d4 = s_bias + CH;
    uint64_t *s_bar = reinterpret_cast<uint64_t *>(smem + S::bar_off);
    long long &s_item = *reinterpret_cast<long long *>(smem + S::item_off);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cl = warp * 8 + (lane >> 2);  // channel within the group
    const int q = lane & 3;                 // state quarter: states q, q+4, q+8, q+12
    const int ntok = p.has_gate ? 3 : 2;
    const uint32_t stage_bytes = uint32_t(ntok * BOX * sizeof(T));
    const T *Bm = static_cast<const T *>(p.Bm);
    const T *Cm = static_cast<const T *>(p.Cm);

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(&s_bar[s], 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_dt);
        if (p.has_gate) prefetch_tensormap(&tm_z);
        prefetch_tensormap(&tm_y);
    }
    __syncthreads();

    uint32_t use_seq = 0;  // TMA loads consumed by this block so far (same on all threads)
    uint32_t y_seq = 0;    // y tiles stored by this block so far

    for (;;) {
        if (tid == 0) s_item = (long long)atomicAdd(p.counter, 1u);
        __syncthreads();
        const long long item = s_item;
        if (item >= p.items) break;
        const int64_t k = item / p.G, g = item % p.G;
        const int64_t b = g / p.Dg, d0 = (g % p.Dg) * CH;
        const int64_t t_beg = k * p.seg_len;
        const int64_t t_end = min(p.L, t_beg + p.seg_len);
        const int ntiles = int((t_end - t_beg + TT - 1) / TT);
        const uint32_t base = use_seq;

        auto issue_load = [&](int j) {  // thread 0 only
            const uint32_t st = (base + j) % STAGES;
            T *dst = s_in + size_t(st) * 3 * BOX;
            const int tt0 = int(t_beg + int64_t(j) * TT);
            mbar_arrive_expect_tx(&s_bar[st], stage_bytes);
            tma_load_3d(dst, &tm_x, &s_bar[st], int(d0), tt0, int(b));
            tma_load_3d(dst + BOX, &tm_dt, &s_bar[st], int(d0), tt0, int(b));
            if (p.has_gate) tma_load_3d(dst + 2 * BOX, &tm_z, &s_bar[st], int(d0), tt0, int(b));
        };
        if (tid == 0)
            for (int j = 0; j < min(STAGES, ntiles); ++j) issue_load(j);

        // Per-lane channel parameters.
        const int64_t d = d0 + cl;
        const bool dvalid = d < p.D;
        float Al[4];
        bool structured = true;
        {
            const float a0 = dvalid ? __ldg(p.A + d * p.N) : 0.f;
            const float del = (dvalid && p.N >= 2) ? __ldg(p.A + d * p.N + 1) - a0 : 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int n = q + 4 * j;
                const float an = (dvalid && n < p.N) ? __ldg(p.A + d * p.N + n) : 0.f;
                Al[j] = an;  // the step's scale Delta * log2(e) is folded into the prologue
                if (dvalid && n < p.N && an != a0 + float(n) * del) structured = false;
            }
        }
        const float Dd = (dvalid && p.Dskip) ? __ldg(p.Dskip + d) : 0.f;
        if (tid < CH) {
            const int64_t dd = d0 + tid;
            const bool ok = dd < p.D;
            s_bias[tid] = (ok && p.dt_bias) ? __ldg(p.dt_bias + dd) : 0.f;
            s_d4[tid] = (ok && p.N >= 2) ? 4.f * (__ldg(p.A + dd * p.N + 1) - __ldg(p.A + dd * p.N)) : 0.f;
        }
        const bool use_struct = __syncthreads_and(structured) && p.allow_structured;

        // Initial state of this segment.
        float h[4];
        if (k == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int n = q + 4 * j;
                h[j] = (dvalid && n < p.N && p.h0) ? __ldg(p.h0 + ((b * p.D + d) * p.N + n)) : 0.f;
            }
        } else {
            if (tid == 0) {
                // The predecessor item (g, k-1) was claimed earlier by a running block.
                if (ld_acquire_gpu(p.flags + g) < uint32_t(k)) {
                    const uint64_t start = globaltimer_ns();
                    for (uint32_t it = 1;; ++it) {
                        if (ld_acquire_gpu(p.flags + g) >= uint32_t(k)) break;
                        __nanosleep(64);
                        if ((it & 63u) == 0 && globaltimer_ns() - start > kWaitLimitNs) {
                            atomicExch(p.status, uint32_t(SSM_ERR_TIMEOUT));
                            break;  // carry on with whatever state is there; the status reports it
                        }
                    }
                }
                __threadfence();
            }
            __syncthreads();
            const float4 hv = __ldcg(reinterpret_cast<const float4 *>(p.carry + (g * CH + cl) * kMaxN + q * 4));
            h[0] = hv.x;
            h[1] = hv.y;
            h[2] = hv.z;
            h[3] = hv.w;
        }

        // B_t / C_t rows of a tile, permuted so that lane q reads states q, q+4, q+8, q+12
        // as one float4: slot s = 4 q + j holds state n = q + 4 j.
        float bcr[BC_PER_THREAD];
        auto fetch_bc = [&](int j) {
            const int64_t tt0 = t_beg + int64_t(j) * TT;
#pragma unroll
            for (int i = 0; i < BC_PER_THREAD; ++i) {
                const int e = tid + i * NT;
                const int t = e >> 5, m = e & 31, sl = m & 15;
                const int n = (sl >> 2) + 4 * (sl & 3);
                const int64_t tt = tt0 + t;
                float v = 0.f;
                if (tt < t_end && n < p.N) {
                    const T *src = (m < 16) ? Bm : Cm;
                    v = Tok<T>::ldg(src + ((b * p.L + tt) * p.N + n));
                }
                bcr[i] = v;
            }
        };
        fetch_bc(0);

        for (int j = 0; j < ntiles; ++j) {
            const int64_t t0 = t_beg + int64_t(j) * TT;
            const int tlen = int(t_end - t0 < TT ? t_end - t0 : TT);
            const uint32_t seq = use_seq++;
            const uint32_t st = seq % STAGES;
            const bool landed = wait_bar(&s_bar[st], (seq / STAGES) & 1u);
            const T *sx = s_in + size_t(st) * 3 * BOX;
            const T *sdt = sx + BOX;
            const T *sz = sx + 2 * BOX;
            // Prologue: once per (t, channel) of the tile.
            for (int e = tid; e < BOX; e += NT) {
                const int t = e / CH, c = e % CH;
                float4 pr = make_float4(0.f, 0.f, 1.f, 0.f);  // neutral step past the end: h unchanged
                if (t < tlen) {
                    const float v = Tok<T>::to_f(sdt[e]) + s_bias[c];
                    const float delta = p.softplus ? softplus_f(v) : v;
                    const float dl = delta * kLog2e;
                    pr = make_float4(delta * Tok<T>::to_f(sx[e]), dl, ex2_approx(dl * s_d4[c]), 0.f);
                }
                s_pro[e] = pr;
            }
#pragma unroll
            for (int i = 0; i < BC_PER_THREAD; ++i) s_bc[tid + i * NT] = bcr[i];
            // One block-wide decision: if any thread's bounded wait for the tile gave up,
            // every thread leaves (the tile's contents were not used for any output).
            if (__syncthreads_or(!landed)) {
                if (tid == 0) atomicExch(p.status, uint32_t(SSM_ERR_TIMEOUT));
                return;
            }
            if (j + 1 < ntiles) fetch_bc(j + 1);

            T *sy = s_y + size_t(y_seq & 1u) * BOX;
            if (use_struct) {
                if (p.has_gate) scan_tile<T, CH, true, true>(s_pro, s_bc, sx, sz, sy, cl, q, Al, Dd, h);
                else scan_tile<T, CH, true, false>(s_pro, s_bc, sx, sz, sy, cl, q, Al, Dd, h);
            } else {
                if (p.has_gate) scan_tile<T, CH, false, true>(s_pro, s_bc, sx, sz, sy, cl, q, Al, Dd, h);
                else scan_tile<T, CH, false, false>(s_pro, s_bc, sx, sz, sy, cl, q, Al, Dd, h);
            }
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) {
                tma_store_3d(&tm_y, sy, int(d0), int(t0), int(b));
                bulk_commit();
                if (j + STAGES < ntiles) issue_load(j + STAGES);
                bulk_wait_read<1>();  // the store that used the other y buffer has read it
            }
            ++y_seq;
        }

        // Hand the state over, or write the final state.
        if (k == p.K - 1) {
            if (p.h_last && dvalid) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int n = q + 4 * j;
                    if (n < p.N) p.h_last[(b * p.D + d) * p.N + n] = h[j];
                }
            }
        } else {
            *reinterpret_cast<float4 *>(p.carry + (g * CH + cl) * kMaxN + q * 4) = make_float4(h[0], h[1], h[2], h[3]);
            __syncthreads();
            if (tid == 0 && !(p.drop_handoff && g == 0 && k == 0)) {
                __threadfence();
                st_release_gpu(p.flags + g, uint32_t(k + 1));
            }
        }
        __syncthreads();
    }
    if (tid == 0) bulk_wait_read<0>();
}

// ------------------------------------------------------------- step kernel
template <typename T>
__global__ void __launch_bounds__(128)
    step_kernel(int64_t Bsz, int64_t D, int N, int softplus, const T *__restrict__ x, const T *__restrict__ dt,
                const T *__restrict__ z, const T *__restrict__ Bm, const T *__restrict__ Cm,
                const float *__restrict__ A, const float *__restrict__ Dskip, const float *__restrict__ dt_bias,
                float *__restrict__ h, T *__restrict__ y) {
    const int64_t ch = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (ch >= Bsz * D) return;
    const int64_t b = ch / D, d = ch % D;
    const float xv = Tok<T>::ldg(x + ch);
    const float v = Tok<T>::ldg(dt + ch) + (dt_bias ? __ldg(dt_bias + d) : 0.f);
    const float delta = softplus ? softplus_f(v) : v;
    const float dl = delta * kLog2e, u = delta * xv;
    float yv = 0.f;
    float *hp = h + ch * N;
    if (N == kMaxN) {
        float4 hv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) hv[i] = reinterpret_cast<const float4 *>(hp)[i];
        float *hs = reinterpret_cast<float *>(hv);
#pragma unroll
        for (int n = 0; n < kMaxN; ++n) {
            const float a = ex2_approx(dl * __ldg(A + d * kMaxN + n));
            hs[n] = fmaf(a, hs[n], u * Tok<T>::ldg(Bm + b * kMaxN + n));
            yv = fmaf(Tok<T>::ldg(Cm + b * kMaxN + n), hs[n], yv);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) reinterpret_cast<float4 *>(hp)[i] = hv[i];
    } else {
        for (int n = 0; n < N; ++n) {
            const float a = ex2_approx(dl * __ldg(A + d * N + n));
            const float hn = fmaf(a, hp[n], u * Tok<T>::ldg(Bm + b * N + n));
            hp[n] = hn;
            yv = fmaf(Tok<T>::ldg(Cm + b * N + n), hn, yv);
        }
    }
    yv = fmaf(Dskip ? __ldg(Dskip + d) : 0.f, xv, yv);
    if (z) yv *= silu_f(Tok<T>::ldg(z + ch));
    y[ch] = Tok<T>::from_f(yv);
}

// ----------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &qres) ==
                cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// [B, L, D] token tensor as a 3-D TMA map with a [CH x TT x 1] box.
bool make_token_map(CUtensorMap *m, const void *ptr, ssm_dtype dt, int64_t Bsz, int64_t L, int64_t D, int ch) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    const size_t es = dt == SSM_BF16 ? 2 : 4;
    cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(L), cuuint64_t(Bsz)};
    cuuint64_t strides[2] = {cuuint64_t(D * es), cuuint64_t(L * D * es)};
    cuuint32_t box[3] = {cuuint32_t(ch), cuuint32_t(TT), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, dt == SSM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                     const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

struct ScanPlan {
    int warps = 4, ch = 32;
    int64_t G = 0, Dg = 0, K = 0, seg_len = 0, items = 0;
    int grid = 0;
    size_t smem = 0;
};

template <typename T, int WARPS>
void *kernel_ptr() {
    return reinterpret_cast<void *>(&scan_fwd_kernel<T, WARPS>);
}
template <typename T, int WARPS>
size_t smem_bytes() {
    return ScanSmem<T, WARPS>::total;
}

void *pick_kernel(ssm_dtype dt, int warps) {
    if (dt == SSM_BF16) return warps == 4 ? kernel_ptr<__nv_bfloat16, 4>() : kernel_ptr<__nv_bfloat16, 2>();
    return warps == 4 ? kernel_ptr<float, 4>() : kernel_ptr<float, 2>();
}
size_t pick_smem(ssm_dtype dt, int warps) {
    if (dt == SSM_BF16) return warps == 4 ? smem_bytes<__nv_bfloat16, 4>() : smem_bytes<__nv_bfloat16, 2>();
    return warps == 4 ? smem_bytes<float, 4>() : smem_bytes<float, 2>();
}

// Largest group count over both block shapes: bounds the flag and state arrays.
int64_t max_groups(int64_t Bsz, int64_t D) { return Bsz * ((D + 15) / 16); }

size_t ws_flags_off() { return kWsHeader; }
size_t ws_carry_off(int64_t Bsz, int64_t D) { return round_up(kWsHeader + size_t(max_groups(Bsz, D)) * 4, 256); }
size_t ws_total(int64_t Bsz, int64_t D) {
    return ws_carry_off(Bsz, D) + size_t(Bsz) * size_t(round_up(size_t(D), 32)) * kMaxN * 4;
}

bool plan_scan(const ssm_scan_args *a, ScanPlan *pl) {
    const int sms = sm_count();
    if (sms <= 0) return false;
    const int64_t G32 = a->batch * ((a->dim + 31) / 32);
    pl->warps = (G32 >= 2 * int64_t(sms)) ? 4 : 2;
    pl->ch = 8 * pl->warps;
    pl->Dg = (a->dim + pl->ch - 1) / pl->ch;
    pl->G = a->batch * pl->Dg;
    pl->smem = pick_smem(a->dtype, pl->warps);
    void *kern = pick_kernel(a->dtype, pl->warps);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(pl->smem)) != cudaSuccess)
        return false;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, pl->warps * 32, pl->smem) != cudaSuccess ||
        occ <= 0)
        return false;
    pl->grid = int(std::min<int64_t>(pl->G, int64_t(occ) * sms));
    // Enough (group, segment) items that the dynamic hand-out balances the blocks.
    const int64_t want_k = std::max<int64_t>(1, (32 * int64_t(pl->grid) + pl->G - 1) / pl->G);
    const int64_t per = (a->seqlen + want_k - 1) / want_k;
    pl->seg_len = std::max<int64_t>(TT, (per + TT - 1) / TT * TT);
    pl->K = (a->seqlen + pl->seg_len - 1) / pl->seg_len;
    pl->items = pl->G * pl->K;
    return true;
}

ssm_status check_common(int64_t Bsz, int64_t D, int64_t N, ssm_dtype dt, uint32_t flags) {
    if (Bsz < 0 || D < 0 || N < 1) return SSM_ERR_INVALID;
    if (dt != SSM_F32 && dt != SSM_BF16) return SSM_ERR_INVALID;
    if (flags & ~uint32_t(SSM_DELTA_SOFTPLUS | SSM_A_GENERAL | SSM_TEST_DROP_HANDOFF)) return SSM_ERR_INVALID;
    if (N > kMaxN) return SSM_ERR_UNSUPPORTED;
    if (D % (dt == SSM_BF16 ? 8 : 4) != 0) return SSM_ERR_UNSUPPORTED;
    return SSM_OK;
}

ssm_status validate_scan(const ssm_scan_args *a) {
    if (!a) return SSM_ERR_INVALID;
    if (a->seqlen < 0) return SSM_ERR_INVALID;
    ssm_status s = check_common(a->batch, a->dim, a->dstate, a->dtype, a->flags);
    if (s != SSM_OK) return s;
    if (a->batch > INT32_MAX || a->seqlen > INT32_MAX || a->dim > INT32_MAX) return SSM_ERR_UNSUPPORTED;
    const bool work = a->batch > 0 && a->dim > 0 && a->seqlen > 0;
    if (work && (!a->x || !a->dt || !a->Bm || !a->Cm || !a->A || !a->y)) return SSM_ERR_INVALID;
    // Tokens moved by TMA and the workspace need 16 bytes; everything else its element size.
    const size_t es = a->dtype == SSM_BF16 ? 2 : 4;
    const void *p16[] = {a->x, a->dt, a->z, a->y, a->workspace};
    for (const void *p : p16)
        if (p && !aligned(p, 16)) return SSM_ERR_UNSUPPORTED;
    const void *pes[] = {a->Bm, a->Cm};
    for (const void *p : pes)
        if (p && !aligned(p, es)) return SSM_ERR_UNSUPPORTED;
    const void *p4[] = {a->A, a->Dskip, a->dt_bias, a->h0, a->h_last};
    for (const void *p : p4)
        if (p && !aligned(p, 4)) return SSM_ERR_UNSUPPORTED;
    if (work && (!a->workspace || a->workspace_bytes < ws_total(a->batch, a->dim))) return SSM_ERR_INVALID;
    return SSM_OK;
}

// ------------------------------------------------ allocation-free variant
// Scratch for ssm_scan_fwd_noalloc: a fixed device array that every GPU which
// loads this library holds until the process exits. 2 MiB covers the hand-over
// state of a little over 32,000 channels (B x D).
constexpr size_t kStaticScratchBytes = size_t(2) << 20;
__device__ __align__(256) unsigned char g_scan_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
unsigned char *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scan_scratch on the current device. The host-side symbol
// is only a stand-in, so the address is looked up once per device (with that
// device current) and cached.
unsigned char *static_scratch() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scan_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_ptr[dev] = static_cast<unsigned char *>(p);
    }
    return g_scratch_ptr[dev];
}

}  // namespace

// ======================================================================= C ABI
extern "C" {

size_t ssm_scan_workspace_size(const ssm_scan_args *a) {
    if (!a || a->batch < 0 || a->dim < 0) return 0;
    return ws_total(a->batch, a->dim);
}

ssm_status ssm_scan_fwd(const ssm_scan_args *a, void *stream_) {
    ssm_status s = validate_scan(a);
    if (s != SSM_OK) return s;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (a->batch == 0 || a->dim == 0) return SSM_OK;
    const size_t hbytes = size_t(a->batch) * a->dim * a->dstate * 4;
    if (a->seqlen == 0) {  // empty sequence: the final state is the initial one
        if (!a->h_last) return SSM_OK;
        cudaError_t e = a->h0 ? cudaMemcpyAsync(a->h_last, a->h0, hbytes, cudaMemcpyDeviceToDevice, stream)
                              : cudaMemsetAsync(a->h_last, 0, hbytes, stream);
        return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
    }
    ScanPlan pl;
    if (!plan_scan(a, &pl)) return SSM_ERR_CUDA;
    unsigned char *ws = static_cast<unsigned char *>(a->workspace);
    // Clear the item counter, the status word and the flags of the groups in use.
    if (cudaMemsetAsync(ws, 0, ws_flags_off() + size_t(pl.G) * 4, stream) != cudaSuccess) return SSM_ERR_CUDA;

    CUtensorMap tx, tdt, tz, ty;
    if (!make_token_map(&tx, a->x, a->dtype, a->batch, a->seqlen, a->dim, pl.ch) ||
        !make_token_map(&tdt, a->dt, a->dtype, a->batch, a->seqlen, a->dim, pl.ch) ||
        !make_token_map(&tz, a->z ? a->z : a->x, a->dtype, a->batch, a->seqlen, a->dim, pl.ch) ||
        !make_token_map(&ty, a->y, a->dtype, a->batch, a->seqlen, a->dim, pl.ch))
        return SSM_ERR_CUDA;

    ScanParams p;
    p.L = a->seqlen;
    p.D = a->dim;
    p.N = a->dstate;
    p.G = pl.G;
    p.Dg = pl.Dg;
    p.K = pl.K;
    p.seg_len = pl.seg_len;
    p.items = pl.items;
    p.Bm = a->Bm;
    p.Cm = a->Cm;
    p.A = a->A;
    p.Dskip = a->Dskip;
    p.dt_bias = a->dt_bias;
    p.h0 = a->h0;
    p.h_last = a->h_last;
    p.counter = reinterpret_cast<uint32_t *>(ws);
    p.status = reinterpret_cast<uint32_t *>(ws + 4);
    p.flags = reinterpret_cast<uint32_t *>(ws + ws_flags_off());
    p.carry = reinterpret_cast<float *>(ws + ws_carry_off(a->batch, a->dim));
    p.has_gate = a->z != nullptr;
    p.softplus = (a->flags & SSM_DELTA_SOFTPLUS) != 0;
    p.allow_structured = (a->flags & SSM_A_GENERAL) == 0;
    p.drop_handoff = (a->flags & SSM_TEST_DROP_HANDOFF) != 0;

    void *kern = pick_kernel(a->dtype, pl.warps);
    void *args[] = {&tx, &tdt, &tz, &ty, &p};
    cudaError_t e = cudaLaunchKernel(kern, dim3(pl.grid), dim3(pl.warps * 32), args, pl.smem, stream);
    return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

ssm_status ssm_step(int64_t batch, int64_t dim, int64_t dstate, ssm_dtype dtype, uint32_t flags, const void *x,
                    const void *dt, const void *z, const void *Bm, const void *Cm, const float *A,
                    const float *Dskip, const float *dt_bias, float *h, void *y, void *stream_) {
    ssm_status s = check_common(batch, dim, dstate, dtype, flags);
    if (s != SSM_OK) return s;
    if (batch == 0 || dim == 0) return SSM_OK;
    if (!x || !dt || !Bm || !Cm || !A || !h || !y) return SSM_ERR_INVALID;
    const size_t es = dtype == SSM_BF16 ? 2 : 4;
    const void *pes[] = {x, dt, z, Bm, Cm, y};
    for (const void *p : pes)
        if (p && !aligned(p, es)) return SSM_ERR_UNSUPPORTED;
    const void *p4[] = {A, Dskip, dt_bias};
    for (const void *p : p4)
        if (p && !aligned(p, 4)) return SSM_ERR_UNSUPPORTED;
    if (!aligned(h, dstate == kMaxN ? 16 : 4)) return SSM_ERR_UNSUPPORTED;  // float4 state rows when N = 16
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const int64_t nch = batch * dim;
    const int threads = 128;
    const int64_t blocks = (nch + threads - 1) / threads;
    if (blocks > INT32_MAX) return SSM_ERR_UNSUPPORTED;
    const int sp = (flags & SSM_DELTA_SOFTPLUS) != 0;
    if (dtype == SSM_BF16) {
        using T = __nv_bfloat16;
        step_kernel<T><<<unsigned(blocks), threads, 0, stream>>>(
            batch, dim, int(dstate), sp, static_cast<const T *>(x), static_cast<const T *>(dt),
            static_cast<const T *>(z), static_cast<const T *>(Bm), static_cast<const T *>(Cm), A, Dskip, dt_bias, h,
            static_cast<T *>(y));
    } else {
        step_kernel<float><<<unsigned(blocks), threads, 0, stream>>>(
            batch, dim, int(dstate), sp, static_cast<const float *>(x), static_cast<const float *>(dt),
            static_cast<const float *>(z), static_cast<const float *>(Bm), static_cast<const float *>(Cm), A, Dskip,
            dt_bias, h, static_cast<float *>(y));
    }
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

ssm_status ssm_workspace_status(const void *workspace, void *stream_) {
    if (!workspace) return SSM_ERR_INVALID;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, static_cast<const unsigned char *>(workspace) + 4, 4, cudaMemcpyDeviceToHost, stream) !=
            cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return SSM_ERR_CUDA;
    return v == 0 ? SSM_OK : static_cast<ssm_status>(v);
}

ssm_status ssm_scan_fwd_noalloc(const ssm_scan_args *a, void *stream) {
    if (!a || a->batch < 0 || a->dim < 0) return SSM_ERR_INVALID;
    if (ws_total(a->batch, a->dim) > kStaticScratchBytes) return SSM_ERR_UNSUPPORTED;
    unsigned char *scratch = static_scratch();
    if (!scratch) return SSM_ERR_CUDA;
    ssm_scan_args b = *a;
    b.workspace = scratch;
    b.workspace_bytes = kStaticScratchBytes;
    return ssm_scan_fwd(&b, stream);
}

const char *ssm_status_string(ssm_status s) {
    switch (s) {
        case SSM_OK: return "SSM_OK";
        case SSM_ERR_INVALID: return "SSM_ERR_INVALID: invalid argument";
        case SSM_ERR_UNSUPPORTED: return "SSM_ERR_UNSUPPORTED: shape, alignment or size not supported";
        case SSM_ERR_CUDA: return "SSM_ERR_CUDA: a CUDA call or launch failed";
        case SSM_ERR_TIMEOUT: return "SSM_ERR_TIMEOUT: a device-side wait for a carried state timed out";
        default: return "unknown ssm_status";
    }
}

}  // extern "C"
