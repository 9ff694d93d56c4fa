// ssm_scan.cu -- host side and C ABI of the B200 (sm_100a) selective state space
// (S6) library: argument checks, workspace layout, TMA descriptors, the launch
// plan of the warp-specialised scan kernel (ssm_scan_kernel.cuh), the one-token
// decode kernel, and the allocation-free scan variant.
//
// Sequence parallelism: the sequence of every group of 32 channels is cut into
// time segments; (group, segment) items are handed out in order by an atomic
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
#include <type_traits>

#include "../../include/ssm_scan.h"
#include "ssm_device.cuh"
#include "ssm_scan_kernel.cuh"

using namespace ssm;


namespace {

constexpr int kMaxN = 16;   // states per channel handled by the kernels
constexpr int kMinSegTiles = 32;  // shortest time segment, in tiles (unless the sequence is shorter)
constexpr int kMaxSegTiles = 256;  // longest time segment, in tiles

// ------------------------------------------------------------- workspace
// [0, 4) item counter; [4, 8) device status; [256, ...) per-group flags;
// then per-group hand-off states float32 [G][CH][16].
constexpr size_t kWsHeader = 256;

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Exact zero-order hold: Bbar / B per unit input = (Abar - 1) / A, by the series
// Delta (1 + z/2 + z^2/6 + z^3/24 + z^4/120), z = Delta A, below |z| = 1/16.
__device__ __forceinline__ float zoh_w(const float delta, const float A, const float abar) {
    const float z = delta * A;
    if (fabsf(z) < 0.0625f)
        return delta * fmaf(z, fmaf(z, fmaf(z, fmaf(z, 1.f / 120.f, 1.f / 24.f), 1.f / 6.f), 0.5f), 1.f);
    return __fdividef(abar - 1.f, A);
}

// The short convolution at one decode step for channel d: u = silu(cb + w.x s0 + w.y s1 +
// w.z s2 + w.w x), s = the three previous tokens of the window (conv_state [B, 3, D],
// oldest first; s points at s0, the others follow at stride D). The same fused
// multiply-adds in the same order as the scan kernel's.
template <typename T>
__device__ __forceinline__ float conv_u(const float xv, const T *s, const int64_t D, const float4 w, const float cb) {
    float v = fmaf(w.x, Tok<T>::to_f(s[0]), cb);
    v = fmaf(w.y, Tok<T>::to_f(s[D]), v);
    v = fmaf(w.z, Tok<T>::to_f(s[2 * D]), v);
    v = fmaf(w.w, xv, v);
    return silu_f(v);
}

// Taps ([D, 4], one float4 per channel) and bias of channel d.
__device__ __forceinline__ float4 conv_taps(const float *w, const int64_t d) {
    return __ldg(reinterpret_cast<const float4 *>(w) + d);
}

// ------------------------------------------------------------- step kernel
// CONV: the SSM's input is the short convolution's u; the window conv_state moves by one
// token (s0, s1, s2) -> (s1, s2, x).
template <typename T, bool ZOH, bool CONV>
__global__ void __launch_bounds__(128)
    step_kernel(int64_t Bsz, int64_t D, int N, int softplus, const T *__restrict__ x, const T *__restrict__ dt,
                const T *__restrict__ z, const T *__restrict__ Bm, const T *__restrict__ Cm,
                const float *__restrict__ A, const float *__restrict__ Dskip, const float *__restrict__ dt_bias,
                float *__restrict__ h, T *__restrict__ y, const float *__restrict__ conv_w,
                const float *__restrict__ conv_b, T *__restrict__ conv_state) {
    const int64_t ch = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (ch >= Bsz * D) return;
    const int64_t b = ch / D, d = ch % D;
    float xv = Tok<T>::ldg(x + ch);
    if (CONV) {
        T *s = conv_state + b * 3 * D + d;
        const T s1 = s[D], s2 = s[2 * D];
        xv = conv_u<T>(xv, s, D, conv_taps(conv_w, d), conv_b ? __ldg(conv_b + d) : 0.f);
        s[0] = s1;
        s[D] = s2;
        s[2 * D] = x[ch];
    }
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
            const float an = __ldg(A + d * kMaxN + n), a = ex2_approx(dl * an);
            const float bx = ZOH ? xv * zoh_w(delta, an, a) : u;
            hs[n] = fmaf(a, hs[n], bx * Tok<T>::ldg(Bm + b * kMaxN + n));
            yv = fmaf(Tok<T>::ldg(Cm + b * kMaxN + n), hs[n], yv);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) reinterpret_cast<float4 *>(hp)[i] = hv[i];
    } else {
        for (int n = 0; n < N; ++n) {
            const float an = __ldg(A + d * N + n), a = ex2_approx(dl * an);
            const float bx = ZOH ? xv * zoh_w(delta, an, a) : u;
            const float hn = fmaf(a, hp[n], bx * Tok<T>::ldg(Bm + b * N + n));
            hp[n] = hn;
            yv = fmaf(Tok<T>::ldg(Cm + b * N + n), hn, yv);
        }
    }
    yv = fmaf(Dskip ? __ldg(Dskip + d) : 0.f, xv, yv);
    if (z) yv *= silu_f(Tok<T>::ldg(z + ch));
    y[ch] = Tok<T>::from_f(yv);
}

// One-token step with N = 16: two threads per channel, thread q owning states 8q ..
// 8q+7 as two float4, so that a warp's loads and stores of h cover 1 KB of contiguous
// state (each 32-byte sector is used whole by the pair of loads); the per-channel
// work (softplus, gate) is repeated by only two threads, and the readout is summed
// with one butterfly shuffle. Requires 16-byte aligned h and A rows and 4-element
// aligned B, C rows.
// CONV as for step_kernel: both threads of a channel form u; the first moves the window
// once both have read it (after the warp-wide shuffle).
template <typename T, bool ZOH, bool CONV>
__global__ void __launch_bounds__(256)
    step_pair_kernel(int64_t Bsz, int64_t D, int softplus, const T *__restrict__ x, const T *__restrict__ dt,
                     const T *__restrict__ z, const T *__restrict__ Bm, const T *__restrict__ Cm,
                     const float *__restrict__ A, const float *__restrict__ Dskip, const float *__restrict__ dt_bias,
                     float *__restrict__ h, T *__restrict__ y, const float *__restrict__ conv_w,
                     const float *__restrict__ conv_b, T *__restrict__ conv_state) {
    const int64_t gid = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t ch = gid >> 1;
    const int q = int(gid & 1);
    const bool valid = ch < Bsz * D;  // both threads of a channel agree
    const int64_t chv = valid ? ch : 0;
    const int64_t b = chv / D, d = chv % D;
    float yv = 0.f, xv = 0.f;
    T s1{}, s2{};  // CONV: the window's next first two tokens
    if (valid) {
        xv = Tok<T>::ldg(x + ch);
        if (CONV) {
            const T *s = conv_state + b * 3 * D + d;
            s1 = s[D];
            s2 = s[2 * D];
            xv = conv_u<T>(xv, s, D, conv_taps(conv_w, d), conv_b ? __ldg(conv_b + d) : 0.f);
        }
        const float v = Tok<T>::ldg(dt + ch) + (dt_bias ? __ldg(dt_bias + d) : 0.f);
        const float delta = softplus ? softplus_f(v) : v;
        const float dl = delta * kLog2e, u = delta * xv;
        float4 *hp = reinterpret_cast<float4 *>(h + ch * kMaxN) + 2 * q;
        float4 hv[2] = {hp[0], hp[1]};
        const float4 *ap = reinterpret_cast<const float4 *>(A + d * kMaxN) + 2 * q;
        const float4 av[2] = {__ldg(ap), __ldg(ap + 1)};
        const float4 bv[2] = {Tok<T>::quad(Bm + b * kMaxN + 8 * q), Tok<T>::quad(Bm + b * kMaxN + 8 * q + 4)};
        const float4 cv[2] = {Tok<T>::quad(Cm + b * kMaxN + 8 * q), Tok<T>::quad(Cm + b * kMaxN + 8 * q + 4)};
        if (ZOH) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float a0 = ex2_approx(dl * av[i].x), a1 = ex2_approx(dl * av[i].y);
                const float a2 = ex2_approx(dl * av[i].z), a3 = ex2_approx(dl * av[i].w);
                hv[i].x = fmaf(a0, hv[i].x, xv * zoh_w(delta, av[i].x, a0) * bv[i].x);
                hv[i].y = fmaf(a1, hv[i].y, xv * zoh_w(delta, av[i].y, a1) * bv[i].y);
                hv[i].z = fmaf(a2, hv[i].z, xv * zoh_w(delta, av[i].z, a2) * bv[i].z);
                hv[i].w = fmaf(a3, hv[i].w, xv * zoh_w(delta, av[i].w, a3) * bv[i].w);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                hv[i].x = fmaf(ex2_approx(dl * av[i].x), hv[i].x, u * bv[i].x);
                hv[i].y = fmaf(ex2_approx(dl * av[i].y), hv[i].y, u * bv[i].y);
                hv[i].z = fmaf(ex2_approx(dl * av[i].z), hv[i].z, u * bv[i].z);
                hv[i].w = fmaf(ex2_approx(dl * av[i].w), hv[i].w, u * bv[i].w);
            }
        }
        hp[0] = hv[0];
        hp[1] = hv[1];
        yv = fmaf(cv[0].x, hv[0].x, fmaf(cv[0].y, hv[0].y, fmaf(cv[0].z, hv[0].z, cv[0].w * hv[0].w)));
        yv += fmaf(cv[1].x, hv[1].x, fmaf(cv[1].y, hv[1].y, fmaf(cv[1].z, hv[1].z, cv[1].w * hv[1].w)));
    }
    yv += __shfl_xor_sync(0xffffffffu, yv, 1);
    if (valid && q == 0) {
        yv = fmaf(Dskip ? __ldg(Dskip + d) : 0.f, xv, yv);
        if (z) yv *= silu_f(Tok<T>::ldg(z + ch));
        y[ch] = Tok<T>::from_f(yv);
        if (CONV) {
            T *s = conv_state + b * 3 * D + d;
            s[0] = s1;
            s[D] = s2;
            s[2 * D] = x[ch];
        }
    }
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

// A [B, L, inner] tensor as a 3-D TMA map with a [box_inner x box_rows x 1] box.
bool make_map_3d(CUtensorMap *m, const void *ptr, ssm_dtype dt, int64_t Bsz, int64_t L, int64_t inner,
                 int box_inner, int box_rows = ssm::scan::TT) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    const size_t es = dt == SSM_BF16 ? 2 : 4;
    cuuint64_t dims[3] = {cuuint64_t(inner), cuuint64_t(L), cuuint64_t(Bsz)};
    cuuint64_t strides[2] = {cuuint64_t(inner * es), cuuint64_t(L * inner * es)};
    cuuint32_t box[3] = {cuuint32_t(box_inner), cuuint32_t(box_rows), 1};
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
    int ch = ssm::scan::CH;
    bool deep = false;
    bool seqpar = false;  // local pass + combine + main pass instead of the hand-off
    int64_t G = 0, Dg = 0, K = 0, seg_len = 0, items = 0;
    int grid = 0;
    size_t smem = 0;
};

// The deep configuration of the short-convolution kernels has four prologue warps.
template <bool CONV>
using DeepFor = typename std::conditional<CONV, ssm::scan::DeepConv, ssm::scan::Deep>::type;

template <bool ZOH, bool CONV>
void *pick_kernel_t(ssm_dtype dt, bool deep, bool seq) {
    using namespace ssm::scan;
    if (seq)  // the sequence-parallel passes: deep rings only
        return dt == SSM_BF16 ? reinterpret_cast<void *>(&scan_ws_kernel<__nv_bfloat16, DeepFor<CONV>, ZOH, CONV, true>)
                              : reinterpret_cast<void *>(&scan_ws_kernel<float, DeepFor<CONV>, ZOH, CONV, true>);
    if (dt == SSM_BF16)
        return deep ? reinterpret_cast<void *>(&scan_ws_kernel<__nv_bfloat16, DeepFor<CONV>, ZOH, CONV>)
                    : reinterpret_cast<void *>(&scan_ws_kernel<__nv_bfloat16, Shallow, ZOH, CONV>);
    return deep ? reinterpret_cast<void *>(&scan_ws_kernel<float, DeepFor<CONV>, ZOH, CONV>)
                : reinterpret_cast<void *>(&scan_ws_kernel<float, Shallow, ZOH, CONV>);
}
// Threads per block of a configuration.
int pick_threads(bool deep, bool conv) {
    using namespace ssm::scan;
    if (!deep) return Shallow::NTHREADS;
    return conv ? DeepConv::NTHREADS : Deep::NTHREADS;
}
// The exact zero-order hold and the short convolution are separate instantiations, so
// the default kernel carries none of their code.
void *pick_kernel(ssm_dtype dt, bool deep, bool zoh, bool conv, bool seq = false) {
    if (conv) return zoh ? pick_kernel_t<true, true>(dt, deep, seq) : pick_kernel_t<false, true>(dt, deep, seq);
    return zoh ? pick_kernel_t<true, false>(dt, deep, seq) : pick_kernel_t<false, false>(dt, deep, seq);
}
template <bool CONV>
size_t pick_smem_t(ssm_dtype dt, bool deep) {
    using namespace ssm::scan;
    if (dt == SSM_BF16)
        return deep ? Layout<__nv_bfloat16, DeepFor<CONV>, CONV>::total : Layout<__nv_bfloat16, Shallow, CONV>::total;
    return deep ? Layout<float, DeepFor<CONV>, CONV>::total : Layout<float, Shallow, CONV>::total;
}
size_t pick_smem(ssm_dtype dt, bool deep, bool conv) {
    return conv ? pick_smem_t<true>(dt, deep) : pick_smem_t<false>(dt, deep);
}
// Prologue warps of a configuration (each writes its own slot of the segment sums).
int pick_np(bool deep, bool conv) {
    using namespace ssm::scan;
    if (!deep) return Shallow::NP;
    return conv ? DeepConv::NP : Deep::NP;
}

// ------------------------------------------------- sequence-parallel combine
// Between the local pass and the main pass of the sequence-parallel evaluation. Over one
// segment k the recurrence is an affine map of the state, h_end = a_k h_start + l_k, with
// a_k = prod_t Abar_t = 2^(A[d,n] sum_t Delta_t log2 e) (the segment's sum from the
// prologue warps' slots) and l_k the end state the local pass reached from zero. Segment
// 0's local pass started from h0, so a_0 = 0 and its l_0 is already exact; the start state
// of segment k is the composition of maps 0 .. k-1 applied to 0. One warp per state
// h[b, d, n]: lane j composes a run of consecutive segments, the lanes' runs are composed
// by a shuffle scan ((a1, b1) then (a2, b2) is (a2 a1, a2 b1 + b2)), and each lane walks
// its run again writing every segment's start state (segment 0's is h0 and not written).
__global__ void __launch_bounds__(256)
    seqpar_combine_kernel(int64_t G, int64_t K, int64_t Dg, int64_t D, int N, int np, const float *__restrict__ A,
                          const float *__restrict__ seg_local, const float *__restrict__ seg_dsum,
                          float *__restrict__ seg_state) {
    constexpr int CH = ssm::scan::CH, CW = ssm::scan::CW;
    const int64_t wid = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= G * CH * 16) return;
    const int n = int(wid & 15), c = int((wid >> 4) % CH);
    const int64_t g = wid / (16 * CH);
    const int64_t d = (g % Dg) * CH + c;
    const bool valid = d < D && n < N;
    const float An = valid ? A[d * N + n] : 0.f;
    const int w = n >> 2, j = n & 3;
    auto at = [&](int64_t k) { return (((g * K + k) * CW + w) * CH + c) * 4 + j; };
    auto factor = [&](int64_t k) {
        if (k == 0) return 0.f;
        float ds = 0.f;
        for (int h = 0; h < np; ++h) ds += seg_dsum[((g * K + k) * 4 + h) * CH + c];
        return exp2f(An * ds);
    };
    const int64_t per = (K + 31) / 32;
    const int64_t k0 = lane * per < K ? lane * per : K, k1 = k0 + per < K ? k0 + per : K;
    float ar = 1.f, br = 0.f;  // the run's map: h -> ar h + br
    for (int64_t k = k0; k < k1; ++k) {
        const float ak = factor(k), lk = valid ? seg_local[at(k)] : 0.f;
        ar *= ak;
        br = fmaf(ak, br, lk);
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float ap = __shfl_up_sync(0xffffffffu, ar, o), bp = __shfl_up_sync(0xffffffffu, br, o);
        if (lane >= o) {
            br = fmaf(ar, bp, br);
            ar *= ap;
        }
    }
    float h = __shfl_up_sync(0xffffffffu, br, 1);  // the state entering this lane's run
    if (lane == 0) h = 0.f;
    for (int64_t k = k0; k < k1; ++k) {
        if (k > 0) seg_state[at(k)] = valid ? h : 0.f;
        const float ak = factor(k), lk = valid ? seg_local[at(k)] : 0.f;
        h = fmaf(ak, h, lk);
    }
}

// Channel slots B x round_up(D, 32) beyond which no workspace is planned: far above any
// shape whose tokens fit in memory, and low enough that no size below overflows 64 bits.
constexpr uint64_t kMaxChannelSlots = uint64_t(1) << 40;

// B x round_up(D, 32), or 0 when B or D is negative or the count exceeds kMaxChannelSlots
// (tested by division, so nothing overflows on the way).
uint64_t channel_slots(int64_t Bsz, int64_t D) {
    if (Bsz <= 0 || D <= 0 || D > INT64_MAX - 31) return 0;
    const uint64_t d32 = (uint64_t(D) + 31) / 32 * 32;
    if (d32 > kMaxChannelSlots / uint64_t(Bsz)) return 0;
    return uint64_t(Bsz) * d32;
}

// Largest group count over both block shapes (groups of 16 or 32 channels): bounds the
// flag and state arrays; at most channel_slots / 16.
size_t max_groups(int64_t Bsz, int64_t D) { return size_t(Bsz) * size_t((D + 15) / 16); }

size_t ws_flags_off() { return kWsHeader; }
size_t ws_carry_off(int64_t Bsz, int64_t D) { return round_up(kWsHeader + max_groups(Bsz, D) * 4, 256); }
// Workspace bytes of the hand-off evaluation over B sequences of D channels; 0 for shapes
// channel_slots refuses (and for B = 0 or D = 0, which need none).
size_t ws_total(int64_t Bsz, int64_t D) {
    const uint64_t slots = channel_slots(Bsz, D);
    if (slots == 0) return 0;
    return ws_carry_off(Bsz, D) + size_t(slots) * kMaxN * 4;
}

// The sequence-parallel evaluation's area after it, for at most kSeqParMaxItems (group,
// segment) items: each item's local end state and true start state ([CW][CH] float4 each)
// and its prologue warps' sums of Delta log2 e ([4][CH] float).
constexpr int64_t kSeqParMaxItems = 1024;
constexpr size_t kSeqParItemState = size_t(ssm::scan::CW) * ssm::scan::CH * 16;
constexpr size_t kSeqParItemDsum = size_t(4) * ssm::scan::CH * 4;
size_t ws_seqpar_off(int64_t Bsz, int64_t D) { return round_up(ws_total(Bsz, D), 256); }
size_t ws_full(int64_t Bsz, int64_t D) {
    const size_t base = ws_total(Bsz, D);
    if (base == 0) return 0;
    return ws_seqpar_off(Bsz, D) + size_t(kSeqParMaxItems) * (2 * kSeqParItemState + kSeqParItemDsum);
}

// Blocks per SM of the shallow and deep kernel configurations for a token type, with or
// without the short convolution, per device (queried once: the attribute calls cost
// microseconds).
bool scan_occupancy(ssm_dtype dt, bool conv, int occ[2]) {
    constexpr int kDevs = 64;
    static std::mutex mu;
    static int cache[kDevs][2][2][2];
    static bool have[kDevs][2][2];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevs) return false;
    const int ti = dt == SSM_BF16 ? 1 : 0, ci = conv ? 1 : 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!have[dev][ti][ci]) {
        int optin = 0;
        if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
        for (int deep = 0; deep < 2; ++deep) {
            void *kern = pick_kernel(dt, deep != 0, false, conv);
            void *kern_zoh = pick_kernel(dt, deep != 0, true, conv);  // same shape and register budget
            const size_t smem = pick_smem(dt, deep != 0, conv);
            int o = 0;
            if (smem <= size_t(optin)) {
                if (deep)  // the sequence-parallel kernels share the deep shape
                    for (int zoh = 0; zoh < 2; ++zoh)
                        if (cudaFuncSetAttribute(pick_kernel(dt, true, zoh != 0, conv, true),
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
                            return false;
                if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess ||
                    cudaFuncSetAttribute(kern_zoh, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
                        cudaSuccess ||
                    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, pick_threads(deep != 0, conv), smem) !=
                        cudaSuccess)
                    return false;
            }
            cache[dev][ti][ci][deep] = o;
        }
        have[dev][ti][ci] = true;
    }
    occ[0] = cache[dev][ti][ci][0];
    occ[1] = cache[dev][ti][ci][1];
    return occ[0] > 0 || occ[1] > 0;
}

bool plan_scan(const ssm_scan_args *a, ScanPlan *pl) {
    constexpr int TT = ssm::scan::TT;
    const int sms = sm_count();
    if (sms <= 0) return false;
    pl->ch = ssm::scan::CH;
    pl->Dg = (a->dim + pl->ch - 1) / pl->ch;
    pl->G = a->batch * pl->Dg;
    // Shallow rings with two blocks per SM when there are enough channel groups to give
    // most SMs two (at least 1.25 per SM); otherwise the deep configuration (one block per
    // SM) if its shared memory fits.
    int occ[2] = {0, 0};
    const bool conv = a->conv_w != nullptr;
    if (!scan_occupancy(a->dtype, conv, occ)) return false;
    // (measured: the deep rings gain ~8% on 160 groups over 148 SMs and nothing on 192)
    const bool shallow_fills = occ[0] >= 2 && 4 * pl->G >= 5 * int64_t(sms);
    pl->deep = occ[1] > 0 && (occ[0] <= 0 || !shallow_fills);
    pl->smem = pick_smem(a->dtype, pl->deep, conv);
    pl->grid = int(std::min<int64_t>(pl->G, int64_t(occ[pl->deep ? 1 : 0]) * sms));
    // Segments: about four items per block, between kMinSegTiles and kMaxSegTiles tiles
    // long. Each item start waits for its predecessor's state (a few microseconds), which
    // bounds them from below; dynamic claiming balances the blocks only if items are short
    // against the whole run, which bounds them from above.
    const int64_t want_k = std::max<int64_t>(1, (4 * int64_t(pl->grid) + pl->G - 1) / pl->G);
    const int64_t per = (a->seqlen + want_k - 1) / want_k;
    const int64_t lmin = std::min<int64_t>((a->seqlen + TT - 1) / TT * TT, int64_t(kMinSegTiles) * TT);
    pl->seg_len = std::min<int64_t>(int64_t(kMaxSegTiles) * TT,
                                    std::max<int64_t>(std::max<int64_t>(TT, lmin), (per + TT - 1) / TT * TT));
    if (a->flags & SSM_TEST_SHORT_SEGMENTS) pl->seg_len = TT;
    pl->K = (a->seqlen + pl->seg_len - 1) / pl->seg_len;
    pl->items = pl->G * pl->K;

    // Sequence-parallel evaluation: when the groups fill at most a quarter of the block
    // slots (it does about twice the work of the hand-off) and the sequence is long, or when
    // the caller asks; only if the workspace has its area and the sequence gives at least
    // two segments.
    const int64_t slots = int64_t(occ[1]) * sms;  // the sequence-parallel passes use the deep rings
    const bool want = occ[1] > 0 && !(a->flags & SSM_SEQ_HANDOFF) &&
                      ((a->flags & SSM_SEQ_PARALLEL) || (4 * pl->G <= slots && a->seqlen >= 64 * TT));
    if (want && a->workspace_bytes >= ws_full(a->batch, a->dim)) {
        // Segments of at least 16 tiles. The number K of segments minimises the two passes'
        // length in waves of equal items, (ceil(G K / slots) + ceil(G (K - 1) / slots)) x the
        // segment length (the smallest such K on ties): e.g. 32 groups on 148 slots take 9
        // segments (288 + 256 items, two waves each) rather than 10 (320 items need three).
        const int64_t kmax = std::min<int64_t>(kSeqParMaxItems / std::max<int64_t>(pl->G, 1),
                                               (a->seqlen + 16 * TT - 1) / (16 * TT));
        int64_t K = 0, seg = 0;
        double best = 0.0;
        for (int64_t k = 2; k <= kmax; ++k) {
            const int64_t sl = ((a->seqlen + k - 1) / k + TT - 1) / TT * TT;
            const int64_t kr = (a->seqlen + sl - 1) / sl;
            if (kr < 2) continue;
            const double cost = double((pl->G * kr + slots - 1) / slots + (pl->G * (kr - 1) + slots - 1) / slots) *
                                double(sl);
            if (K == 0 || cost < best) {
                best = cost;
                K = kr;
                seg = sl;
            }
        }
        if (a->flags & SSM_TEST_SHORT_SEGMENTS) {
            seg = TT;
            K = (a->seqlen + seg - 1) / seg;
        }
        if (K >= 2 && pl->G * K <= kSeqParMaxItems) {
            pl->seqpar = true;
            pl->deep = true;
            pl->smem = pick_smem(a->dtype, true, conv);
            pl->seg_len = seg;
            pl->K = K;
            pl->items = pl->G * K;
            pl->grid = int(std::min<int64_t>(pl->items, slots));
        }
    }
    return true;
}

ssm_status check_common(int64_t Bsz, int64_t D, int64_t N, ssm_dtype dt, uint32_t flags) {
    if (Bsz < 0 || D < 0 || N < 1) return SSM_ERR_INVALID;
    if (dt != SSM_F32 && dt != SSM_BF16) return SSM_ERR_INVALID;
    if (flags & ~uint32_t(SSM_DELTA_SOFTPLUS | SSM_A_GENERAL | SSM_EXACT_ZOH | SSM_SEQ_PARALLEL |
                          SSM_SEQ_HANDOFF | SSM_TEST_SHORT_SEGMENTS | SSM_TEST_DROP_HANDOFF))
        return SSM_ERR_INVALID;
    if ((flags & SSM_SEQ_PARALLEL) && (flags & SSM_SEQ_HANDOFF)) return SSM_ERR_INVALID;
    if (N > kMaxN) return SSM_ERR_UNSUPPORTED;
    if (D % (dt == SSM_BF16 ? 8 : 4) != 0) return SSM_ERR_UNSUPPORTED;
    return SSM_OK;
}

// Shapes, flags, pointers and alignment of a scan; the workspace is checked separately.
ssm_status validate_shapes(const ssm_scan_args *a) {
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
    const void *p4[] = {a->A, a->Dskip, a->dt_bias, a->h0, a->h_last, a->conv_b};
    for (const void *p : p4)
        if (p && !aligned(p, 4)) return SSM_ERR_UNSUPPORTED;
    // The short convolution: taps read as one float4 per channel; bias and prefix only with taps.
    if (!a->conv_w && (a->conv_b || a->conv_x0)) return SSM_ERR_INVALID;
    if (a->conv_w && !aligned(a->conv_w, 16)) return SSM_ERR_UNSUPPORTED;
    if (a->conv_x0 && !aligned(a->conv_x0, es)) return SSM_ERR_UNSUPPORTED;
    if (a->batch > 0 && a->dim > 0 && channel_slots(a->batch, a->dim) == 0) return SSM_ERR_UNSUPPORTED;
    return SSM_OK;
}

ssm_status validate_scan(const ssm_scan_args *a) {
    const ssm_status s = validate_shapes(a);
    if (s != SSM_OK) return s;
    const bool work = a->batch > 0 && a->dim > 0 && a->seqlen > 0;
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
namespace {

template <typename T, bool ZOH, bool CONV>
void launch_step(bool pair, unsigned grid, int threads, cudaStream_t stream, int64_t batch, int64_t dim, int N,
                 int sp, const void *x, const void *dt, const void *z, const void *Bm, const void *Cm,
                 const float *A, const float *Dskip, const float *dt_bias, float *h, void *y, const float *conv_w,
                 const float *conv_b, void *conv_state) {
    if (pair)
        step_pair_kernel<T, ZOH, CONV><<<grid, threads, 0, stream>>>(
            batch, dim, sp, static_cast<const T *>(x), static_cast<const T *>(dt), static_cast<const T *>(z),
            static_cast<const T *>(Bm), static_cast<const T *>(Cm), A, Dskip, dt_bias, h, static_cast<T *>(y),
            conv_w, conv_b, static_cast<T *>(conv_state));
    else
        step_kernel<T, ZOH, CONV><<<grid, threads, 0, stream>>>(
            batch, dim, N, sp, static_cast<const T *>(x), static_cast<const T *>(dt), static_cast<const T *>(z),
            static_cast<const T *>(Bm), static_cast<const T *>(Cm), A, Dskip, dt_bias, h, static_cast<T *>(y),
            conv_w, conv_b, static_cast<T *>(conv_state));
}

// The exact zero-order hold and the short convolution are separate instantiations.
template <typename T>
void dispatch_step(bool zoh, bool conv, bool pair, unsigned grid, int threads, cudaStream_t stream, int64_t batch,
                   int64_t dim, int N, int sp, const void *x, const void *dt, const void *z, const void *Bm,
                   const void *Cm, const float *A, const float *Dskip, const float *dt_bias, float *h, void *y,
                   const float *conv_w, const float *conv_b, void *conv_state) {
    if (conv) {
        if (zoh)
            launch_step<T, true, true>(pair, grid, threads, stream, batch, dim, N, sp, x, dt, z, Bm, Cm, A, Dskip,
                                       dt_bias, h, y, conv_w, conv_b, conv_state);
        else
            launch_step<T, false, true>(pair, grid, threads, stream, batch, dim, N, sp, x, dt, z, Bm, Cm, A, Dskip,
                                        dt_bias, h, y, conv_w, conv_b, conv_state);
    } else {
        if (zoh)
            launch_step<T, true, false>(pair, grid, threads, stream, batch, dim, N, sp, x, dt, z, Bm, Cm, A, Dskip,
                                        dt_bias, h, y, nullptr, nullptr, nullptr);
        else
            launch_step<T, false, false>(pair, grid, threads, stream, batch, dim, N, sp, x, dt, z, Bm, Cm, A, Dskip,
                                         dt_bias, h, y, nullptr, nullptr, nullptr);
    }
}

// Checks and launch of one decode step; conv_w == NULL: no short convolution.
ssm_status step_impl(int64_t batch, int64_t dim, int64_t dstate, ssm_dtype dtype, uint32_t flags, const void *x,
                     const void *dt, const void *z, const void *Bm, const void *Cm, const float *A,
                     const float *Dskip, const float *dt_bias, const float *conv_w, const float *conv_b,
                     void *conv_state, float *h, void *y, void *stream_) {
    ssm_status s = check_common(batch, dim, dstate, dtype, flags);
    if (s != SSM_OK) return s;
    if (batch == 0 || dim == 0) return SSM_OK;
    if (!x || !dt || !Bm || !Cm || !A || !h || !y) return SSM_ERR_INVALID;
    const bool conv = conv_w != nullptr;
    if (conv && !conv_state) return SSM_ERR_INVALID;
    const size_t es = dtype == SSM_BF16 ? 2 : 4;
    const void *pes[] = {x, dt, z, Bm, Cm, y, conv_state};
    for (const void *p : pes)
        if (p && !aligned(p, es)) return SSM_ERR_UNSUPPORTED;
    const void *p4[] = {A, Dskip, dt_bias, conv_b};
    for (const void *p : p4)
        if (p && !aligned(p, 4)) return SSM_ERR_UNSUPPORTED;
    if (conv && !aligned(conv_w, 16)) return SSM_ERR_UNSUPPORTED;
    if (!aligned(h, dstate == kMaxN ? 16 : 4)) return SSM_ERR_UNSUPPORTED;  // float4 state rows when N = 16
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const int64_t nch = batch * dim;
    const int sp = (flags & SSM_DELTA_SOFTPLUS) != 0;
    const bool zoh = (flags & SSM_EXACT_ZOH) != 0;
    // Two threads per channel when the state rows are whole float4 rows and B, C rows
    // can be read four elements at a time; one thread per channel otherwise.
    const bool pair = dstate == kMaxN && aligned(A, 16) && aligned(Bm, 4 * es) && aligned(Cm, 4 * es);
    const int threads = pair ? 256 : 128;
    const int64_t blocks = ((pair ? 2 : 1) * nch + threads - 1) / threads;
    if (blocks > INT32_MAX) return SSM_ERR_UNSUPPORTED;
    const unsigned grid = unsigned(blocks);
    if (dtype == SSM_BF16)
        dispatch_step<__nv_bfloat16>(zoh, conv, pair, grid, threads, stream, batch, dim, int(dstate), sp, x, dt, z,
                                     Bm, Cm, A, Dskip, dt_bias, h, y, conv_w, conv_b, conv_state);
    else
        dispatch_step<float>(zoh, conv, pair, grid, threads, stream, batch, dim, int(dstate), sp, x, dt, z, Bm, Cm,
                             A, Dskip, dt_bias, h, y, conv_w, conv_b, conv_state);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}


}  // namespace

extern "C" {

size_t ssm_scan_workspace_size(const ssm_scan_args *a) {
    if (!a || a->batch < 0 || a->dim < 0) return 0;
    return ws_full(a->batch, a->dim);
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

    const int es = a->dtype == SSM_BF16 ? 2 : 4;
    const bool bc_tma = (a->dstate * es) % 16 == 0 && aligned(a->Bm, 16) && aligned(a->Cm, 16);
    CUtensorMap tx, tdt, tz, ty, tb, tc;
    const bool conv = a->conv_w != nullptr;
    // With the short convolution the x box carries the three rows before its tile.
    const int x_rows = ssm::scan::TT + (conv ? ssm::scan::KCONV - 1 : 0);
    if (!make_map_3d(&tx, a->x, a->dtype, a->batch, a->seqlen, a->dim, pl.ch, x_rows) ||
        !make_map_3d(&tdt, a->dt, a->dtype, a->batch, a->seqlen, a->dim, pl.ch) ||
        !make_map_3d(&tz, a->z ? a->z : a->x, a->dtype, a->batch, a->seqlen, a->dim, pl.ch) ||
        !make_map_3d(&ty, a->y, a->dtype, a->batch, a->seqlen, a->dim, pl.ch))
        return SSM_ERR_CUDA;
    if (bc_tma) {
        if (!make_map_3d(&tb, a->Bm, a->dtype, a->batch, a->seqlen, a->dstate, kMaxN) ||
            !make_map_3d(&tc, a->Cm, a->dtype, a->batch, a->seqlen, a->dstate, kMaxN))
            return SSM_ERR_CUDA;
    } else {
        tb = tx;  // unused: B and C rows are read with plain loads
        tc = tx;
    }

    ssm::scan::Params p;
    p.Bsz = a->batch;
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
    p.conv_w = a->conv_w;
    p.conv_b = a->conv_b;
    p.conv_x0 = a->conv_x0;
    p.has_gate = a->z != nullptr;
    p.softplus = (a->flags & SSM_DELTA_SOFTPLUS) != 0;
    p.allow_structured = (a->flags & SSM_A_GENERAL) == 0;
    p.drop_handoff = (a->flags & SSM_TEST_DROP_HANDOFF) != 0;
    p.bc_tma = bc_tma;
    p.mode = ssm::scan::kModeHandoff;
    p.item_base = 0;
    p.seg_local = p.seg_state = p.seg_dsum = nullptr;

    void *kern = pick_kernel(a->dtype, pl.deep, (a->flags & SSM_EXACT_ZOH) != 0, conv, pl.seqpar);
    void *args[] = {&tx, &tdt, &tz, &tb, &tc, &ty, &p};
    const int threads = pick_threads(pl.deep, conv);
    if (!pl.seqpar) {
        cudaError_t e = cudaLaunchKernel(kern, dim3(pl.grid), dim3(threads), args, pl.smem, stream);
        return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
    }
    // Sequence-parallel: local pass, combine, main pass over segments 1 .. K-1 (segment 0's
    // outputs come from the local pass, which started it from h0).
    unsigned char *sp = ws + ws_seqpar_off(a->batch, a->dim);
    p.seg_local = reinterpret_cast<float *>(sp);
    p.seg_state = reinterpret_cast<float *>(sp + size_t(kSeqParMaxItems) * kSeqParItemState);
    p.seg_dsum = reinterpret_cast<float *>(sp + size_t(kSeqParMaxItems) * 2 * kSeqParItemState);
    p.mode = ssm::scan::kModeLocal;
    if (cudaLaunchKernel(kern, dim3(pl.grid), dim3(threads), args, pl.smem, stream) != cudaSuccess)
        return SSM_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, 4, stream) != cudaSuccess) return SSM_ERR_CUDA;  // the item counter
    const int64_t warps = pl.G * ssm::scan::CH * 16;
    seqpar_combine_kernel<<<unsigned((warps + 7) / 8), 256, 0, stream>>>(
        pl.G, pl.K, pl.Dg, a->dim, int(a->dstate), pick_np(pl.deep, conv), a->A, p.seg_local, p.seg_dsum,
        p.seg_state);
    if (cudaGetLastError() != cudaSuccess) return SSM_ERR_CUDA;
    p.mode = ssm::scan::kModeFromCarry;
    p.item_base = pl.G;
    const int grid2 = int(std::min<int64_t>(pl.items - pl.G, int64_t(pl.grid)));
    cudaError_t e = cudaLaunchKernel(kern, dim3(grid2), dim3(threads), args, pl.smem, stream);
    return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

ssm_status ssm_step(int64_t batch, int64_t dim, int64_t dstate, ssm_dtype dtype, uint32_t flags, const void *x,
                    const void *dt, const void *z, const void *Bm, const void *Cm, const float *A,
                    const float *Dskip, const float *dt_bias, float *h, void *y, void *stream) {
    return step_impl(batch, dim, dstate, dtype, flags, x, dt, z, Bm, Cm, A, Dskip, dt_bias, nullptr, nullptr, nullptr,
                     h, y, stream);
}

ssm_status ssm_step_conv(int64_t batch, int64_t dim, int64_t dstate, ssm_dtype dtype, uint32_t flags,
                         const void *x, const void *dt, const void *z, const void *Bm, const void *Cm,
                         const float *A, const float *Dskip, const float *dt_bias, const float *conv_w,
                         const float *conv_b, void *conv_state, float *h, void *y, void *stream) {
    if (!conv_w) return SSM_ERR_INVALID;
    return step_impl(batch, dim, dstate, dtype, flags, x, dt, z, Bm, Cm, A, Dskip, dt_bias, conv_w, conv_b,
                     conv_state, h, y, stream);
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
    const ssm_status v = validate_shapes(a);  // before any size arithmetic on the shape
    if (v != SSM_OK) return v;
    if (ws_total(a->batch, a->dim) > kStaticScratchBytes) return SSM_ERR_UNSUPPORTED;
    unsigned char *scratch = static_scratch();
    if (!scratch) return SSM_ERR_CUDA;
    ssm_scan_args b = *a;
    b.workspace = scratch;
    b.workspace_bytes = kStaticScratchBytes;
    return ssm_scan_fwd(&b, stream);
}

ssm_status ssm_noalloc_status(void *stream_) {
    if (!static_scratch()) return SSM_ERR_CUDA;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    uint32_t v = 0;  // the status word sits 4 bytes into the array, as in a caller's workspace
    if (cudaMemcpyFromSymbolAsync(&v, g_scan_scratch, 4, 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return SSM_ERR_CUDA;
    return v == 0 ? SSM_OK : static_cast<ssm_status>(v);
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
