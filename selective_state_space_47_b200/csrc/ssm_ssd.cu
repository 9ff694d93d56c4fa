// ssm_ssd.cu -- the state space model with one scalar A per head (the Mamba-2 restriction)
// in its chunked matrix form on the sm_100a tensor cores (tcgen05 + TMEM), behind
// ssm_ssd_fwd.
//
// Per head h (channels p < P = 64 of the head share its step size and A), state n < N =
// 128, the scan h_t[p, n] = exp(Delta_t A_h) h_{t-1}[p, n] + Delta_t B_t[n] x_t[p],
// y_t[p] = sum_n C_t[n] h_t[p, n] + D_h x_t[p] (times silu(z_t[p]) when z is given) is,
// over a chunk of Q = 128 steps with a_t = A_h (Delta_1 + ... + Delta_t) from the chunk's
// start, the lower-triangular semiseparable matrix product of the structured state space
// duality (Mamba-2 article, mugbit.ir, "Mamba-2 / SSD" section: the recurrence as a
// structured matrix product computed by matrix multiplications on tensor cores):
//
//   G     = C B^T                                   [Q x Q]     (tensor cores)
//   M     = G o exp(a_t - a_s) Delta_s [s <= t]                  (threads, bfloat16)
//   y     = M X + diag(exp(a_t)) C S + D_h X        [Q x P]     (tensor cores; D X in float32)
//   S'    = exp(a_Q) S + B^T diag(exp(a_Q - a_s) Delta_s) X   [N x P] (tensor cores)
//
// where S[n, p] is the state at the chunk's start. Every product is a 128-row tcgen05.mma
// (kind::f16, bfloat16 operands from shared memory, float32 accumulators in tensor memory):
// G 128x128x128, C S 128x64x128 (twice: S in two bfloat16 parts), M X 128x64x128, B^T (w X)
// 128x64x128.
//
// Work decomposition: one persistent block per SM claims (sequence, head, segment) items in
// order; a segment of SEG chunks starts from the state its predecessor segment published
// (bounded release/acquire wait, as in the scan kernel), so the blocks stay balanced for
// any number of heads. Within an item, the B, C and x tiles of the next chunk are loaded
// by TMA while the current chunk is computed.
#include <cudaTypedefs.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "../../include/ssm_scan.h"
#include "ssm_device.cuh"

namespace ssm {
namespace ssd {

constexpr int Q = 128;        // chunk length (rows of every MMA)
constexpr int NS = 128;       // states per head
constexpr int P = 64;         // channels per head
constexpr int NQ = 4;         // column quarters: each row is split between four warps
constexpr int PH = P / NQ;    // channels (columns) per thread
constexpr int PC = PH / 8;    // 16-byte chunks (8 bfloat16) of them
constexpr int NTHREADS = 128 * NQ;  // 16 warps; warp w owns tensor-memory lanes (rows) 32 (w mod 4) .. +31
constexpr int SEG = 16;       // chunks per segment (2048 steps)
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Shared memory (every tile 1024-byte aligned: the 128-byte swizzle repeats every 8 rows).
// A [rows][128 columns] bfloat16 tile is stored as two [rows][64] blocks of 128-byte rows.
constexpr uint32_t kTile128 = Q * 128 * 2;  // 32 KB: [128][128] bf16
constexpr uint32_t kTile64 = Q * 64 * 2;    // 16 KB: [128][64] bf16
constexpr uint32_t OFF_B = 0;                        // B chunk [t][n], two buffers
constexpr uint32_t OFF_C = OFF_B + 2 * kTile128;     // C chunk [t][n], two buffers
constexpr uint32_t OFF_X = OFF_C + 2 * kTile128;     // x chunk [t][p], two buffers
constexpr uint32_t OFF_M = OFF_X + 2 * kTile64;      // M [t][s]
constexpr uint32_t OFF_S = OFF_M + kTile128;         // S [n][p] bfloat16, high part (operand of C S)
constexpr uint32_t OFF_SLO = OFF_S + kTile64;        // S - high part, rounded to bfloat16 again
constexpr uint32_t OFF_MISC = OFF_SLO + kTile64;
constexpr uint32_t OFF_ALPHA = OFF_MISC;             // a_t log2 e per row [Q] f32
constexpr uint32_t OFF_DELTA = OFF_ALPHA + Q * 4;    // Delta_t [Q] f32
constexpr uint32_t OFF_WSUM = OFF_DELTA + Q * 4;     // per-warp sums of the first-quarter warps [4] f32
constexpr uint32_t OFF_BAR = OFF_WSUM + 64;          // mbarriers: load[2], mma
constexpr uint32_t OFF_TMEM = OFF_BAR + 64;          // tensor-memory base address
constexpr uint32_t OFF_ITEM = OFF_TMEM + 16;         // claimed item
constexpr uint32_t SMEM_BYTES = OFF_ITEM + 16 + 1024;  // + slack to align the base to 1024
constexpr uint32_t kLoadBytes = 2 * kTile128 + kTile64;  // one chunk: B, C, x

// Tensor memory: 256 columns x 128 lanes of float32.
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t TM_G = 0, TM_S = 0, TM_YOFF = 128, TM_YDIAG = 192;

struct Params {
    int64_t Bsz, L, H, nchunks, K, items;  // K: segments per sequence
    const __nv_bfloat16 *dt, *z;
    __nv_bfloat16 *y;
    const float *A, *Dskip, *dt_bias, *h0;
    float *h_last;
    uint32_t *counter, *status, *flags;
    float *carry;  // [B*H][NS][P]
    int softplus;
};

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor of a 128-byte-swizzled operand: start address, leading
// and stride byte offsets (16-byte units), descriptor version 1 (bit 46), swizzle mode 2.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
           (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
// Instruction descriptor: bfloat16 A and B, float32 accumulator, M x N, operand majors
// (0: K-major, 1: M/N-major).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
           (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// 32 consecutive float32 columns of this thread's lane (its warp's 32 lanes, 32x32b shape).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 consecutive float32 columns of this thread's lane (32x32b shape).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Bounded wait on phase `parity` of an mbarrier (every thread); false if it gave up.
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - start > kWaitLimitNs) return false;
    return true;
}

// Byte offset of 16-byte chunk j (8 bfloat16) of row r in a [rows][64] block with the
// 128-byte swizzle (the chunk index XOR the row index modulo 8).
__device__ __forceinline__ uint32_t sw_off(int r, int j) { return uint32_t(r) * 128u + uint32_t((j ^ (r & 7)) << 4); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Global loads issued where they stand (volatile): their results are consumed much later in
// the chunk, so their latency must not be moved next to the use.
__device__ __forceinline__ uint16_t ldg_u16_early(const void *p) {
    uint16_t v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint4 ldg_v4_early(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// silu(z) = z / (1 + e^-z) with one special-function-unit operation: the exponential there,
// the reciprocal of d = 1 + e^-z by Newton's method from a seed taken from d's bits
// (0x7EF311C2 minus them: at most 5% relative error, the constant chosen to minimise that
// over a binade) and three steps r <- r + r (1 - d r) (6e-8). -z log2 e is clamped at 125,
// which keeps d inside the seed's range; silu(z) is then z 2^-125, zero to float precision.
__device__ __forceinline__ float silu_1sfu(float z) {
    const float d = 1.0f + ex2_approx(fminf(-z * kLog2e, 125.f));
    float r = __int_as_float(0x7EF311C2 - __float_as_int(d));
#pragma unroll
    for (int i = 0; i < 3; ++i) r = fmaf(r, fmaf(-d, r, 1.f), r);
    return z * r;
}

__device__ __forceinline__ void sts128(uint32_t saddr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t saddr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(saddr)
                 : "memory");
    return v;
}

// ----------------------------------------------------------------- kernel
__global__ void __launch_bounds__(NTHREADS, 1)
    ssd_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
               const __grid_constant__ CUtensorMap tm_x, const Params p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    float *alpha = reinterpret_cast<float *>(smem + OFF_ALPHA);
    float *dlt = reinterpret_cast<float *>(smem + OFF_DELTA);
    float *wsum = reinterpret_cast<float *>(smem + OFF_WSUM);
    uint64_t *bar_load = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *bar_mma = bar_load + 2;   // the MMAs thread 0 issues
    uint64_t *bar_yoff = bar_load + 3;  // Y_off, issued by thread 128 beside thread 0's G
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_TMEM);
    int *item_slot = reinterpret_cast<int *>(smem + OFF_ITEM);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Row (tensor-memory lane) and column quarter qt of this thread: warps w, w+4, w+8, w+12
    // share the lanes 32 (w mod 4) .. +31, warp w + 4 qt taking quarter qt of every row.
    const int row = tid & (Q - 1), qt = tid >> 7, quarter = warp & 3;

    if (tid == 0) {
        mbar_init(&bar_load[0], 1);
        mbar_init(&bar_load[1], 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_yoff, 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_b);
        prefetch_tensormap(&tm_c);
        prefetch_tensormap(&tm_x);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tlane = uint32_t(quarter * 32) << 16;  // this warp's lane block in tensor-memory addresses
    uint32_t ph_load[2] = {0, 0}, ph_mma = 0, ph_yoff = 0;
    bool ok = true;  // every wait of this thread so far completed

    auto mma_wait = [&]() {
        if (!wait_phase(bar_mma, ph_mma)) ok = false;
        ph_mma ^= 1u;
        tc_fence_after();
    };

    for (;;) {
        if (tid == 0) *item_slot = int(atomicAdd(p.counter, 1u));
        __syncthreads();
        const int64_t it = *item_slot;
        if (it >= p.items) break;
        const int64_t bh = it % (p.Bsz * p.H), k = it / (p.Bsz * p.H);
        const int b = int(bh / p.H), h = int(bh % p.H);
        const int64_t c0 = k * SEG, c1 = c0 + SEG < p.nchunks ? c0 + SEG : p.nchunks;
        const float A2 = __ldg(p.A + h) * kLog2e;  // A log2 e
        const float bias = p.dt_bias ? __ldg(p.dt_bias + h) : 0.f;
        const float dskip = p.Dskip ? __ldg(p.Dskip + h) : 0.f;

        // The state at the segment's start: this thread holds S[row][PH qt .. +PH) in float32.
        float S[PH];
        if (k == 0) {
#pragma unroll
            for (int q = 0; q < PH; ++q)
                S[q] = p.h0 ? __ldg(p.h0 + ((int64_t(b) * p.H + h) * P + PH * qt + q) * NS + row) : 0.f;
        } else {
            if (tid == 0 && ld_acquire_gpu(p.flags + bh) < uint32_t(k)) {
                const uint64_t start = globaltimer_ns();
                for (uint32_t n = 1;; ++n) {
                    if (ld_acquire_gpu(p.flags + bh) >= uint32_t(k)) break;
                    __nanosleep(256);
                    if ((n & 63u) == 0 && globaltimer_ns() - start > kWaitLimitNs) {
                        atomicExch(p.status, uint32_t(SSM_ERR_TIMEOUT));
                        break;
                    }
                }
            }
            __syncthreads();
            __threadfence();
            const float4 *src = reinterpret_cast<const float4 *>(p.carry + (bh * NS + row) * P + PH * qt);
#pragma unroll
            for (int q = 0; q < PH / 4; ++q) {
                const float4 v = __ldcg(src + q);
                S[4 * q] = v.x;
                S[4 * q + 1] = v.y;
                S[4 * q + 2] = v.z;
                S[4 * q + 3] = v.w;
            }
        }
        // S as the operand of C S: row n, 64 p contiguous (N-major, 128-byte swizzle), in two
        // bfloat16 parts, S = hi + lo to about 2^-17, so that C S keeps the float32 state's precision
        auto store_S = [&]() {
#pragma unroll
            for (int j = 0; j < PC; ++j) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    hi[e] = pack_bf16(S[8 * j + 2 * e], S[8 * j + 2 * e + 1]);
                    const float2 r = unpack_bf16(hi[e]);
                    lo[e] = pack_bf16(S[8 * j + 2 * e] - r.x, S[8 * j + 2 * e + 1] - r.y);
                }
                sts128(sbase + OFF_S + sw_off(row, PC * qt + j), make_uint4(hi[0], hi[1], hi[2], hi[3]));
                sts128(sbase + OFF_SLO + sw_off(row, PC * qt + j), make_uint4(lo[0], lo[1], lo[2], lo[3]));
            }
        };
        store_S();

        // TMA loads of chunk c into buffer `buf`: B and C as two 64-column boxes each, x one.
        auto issue_loads = [&](int64_t c, int buf) {
            const int t0 = int(c * Q);
            mbar_arrive_expect_tx(&bar_load[buf], kLoadBytes);
            unsigned char *bb = smem + OFF_B + buf * kTile128, *cc = smem + OFF_C + buf * kTile128;
            tma_load_3d(bb, &tm_b, &bar_load[buf], 0, t0, b);
            tma_load_3d(bb + kTile64, &tm_b, &bar_load[buf], 64, t0, b);
            tma_load_3d(cc, &tm_c, &bar_load[buf], 0, t0, b);
            tma_load_3d(cc + kTile64, &tm_c, &bar_load[buf], 64, t0, b);
            tma_load_3d(smem + OFF_X + buf * kTile64, &tm_x, &bar_load[buf], h * P, t0, b);
        };
        // G = C B^T and Y_off = C S of chunk c (buffer buf), once its tiles have landed and S is
        // in shared memory: issued as soon as possible, ahead of the chunk's own work
        auto issue_G_Yoff = [&](int buf) {
            if (!wait_phase(&bar_load[buf], ph_load[buf])) ok = false;
            ph_load[buf] ^= 1u;
            if (tid == 0) {
                tc_fence_after();
                const uint32_t sB = sbase + OFF_B + buf * kTile128, sC = sbase + OFF_C + buf * kTile128;
                constexpr uint32_t iG = idesc_bf16(128, 128, 0, 0);
#pragma unroll
                for (int kk = 0; kk < NS / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * kTile64 + (kk & 3) * 32;  // K block, 32 bytes per 16 columns
                    umma(tmem + TM_G, sw128_desc(sC + koff, 16, 1024), sw128_desc(sB + koff, 16, 1024), iG, kk > 0);
                }
                umma_commit(bar_mma);
            } else if (tid == 128) {  // another warp issues C S at the same time (a thread's MMA issue waits)
                tc_fence_after();
                const uint32_t sC = sbase + OFF_C + buf * kTile128;
                const uint32_t sS = sbase + OFF_S;
                constexpr uint32_t iO = idesc_bf16(128, 64, 0, 1);
#pragma unroll
                for (int kk = 0; kk < 2 * (NS / 16); ++kk) {  // C S_hi, then C S_lo into the same accumulator
                    const int k8 = kk & 7;
                    const uint32_t koff = (k8 >> 2) * kTile64 + (k8 & 3) * 32;
                    const uint32_t sPart = kk < 8 ? sS : sbase + OFF_SLO;
                    umma(tmem + TM_YOFF, sw128_desc(sC + koff, 16, 1024), sw128_desc(sPart + k8 * 2048, kTile64, 1024),
                         iO, kk > 0);
                }
                umma_commit(bar_yoff);
            }
        };
        if (tid == 0) issue_loads(c0, 0);
        // make S (written by threads) visible to the tensor cores before the first C S
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        issue_G_Yoff(0);

        // dt of this thread's row for the first chunk (prefetched one chunk ahead; first quarter)
        const __nv_bfloat16 *dtp = p.dt + (int64_t(b) * p.L) * p.H + h;
        auto load_dt = [&](int64_t c) -> float {
            const int64_t t = c * Q + row;
            return (qt == 0 && t < p.L) ? __uint_as_float(uint32_t(ldg_u16_early(dtp + t * p.H)) << 16) : 0.f;
        };
        float dt_next = load_dt(c0);

        for (int64_t c = c0; c < c1; ++c) {
            const int buf = int((c - c0) & 1);
            const int64_t t0 = c * Q;
            const int64_t trow = t0 + row;
            const bool rvalid = trow < p.L;
            // the next chunk's loads go into the other buffer, whose last readers (the
            // previous chunk's MMAs) have completed
            if (tid == 0 && c + 1 < c1) issue_loads(c + 1, buf ^ 1);
            const float dtv = dt_next;
            if (c + 1 < c1) dt_next = load_dt(c + 1);
            // z of this row's column quarter (the gate), read early so its latency overlaps the MMAs
            uint4 zr[PC];
            if (p.z && rvalid) {
                const uint4 *zp = reinterpret_cast<const uint4 *>(p.z + (int64_t(b) * p.L + trow) * (p.H * P) + h * P);
#pragma unroll
                for (int j = 0; j < PC; ++j) zr[j] = ldg_v4_early(zp + PC * qt + j);
            }

            // Delta and the running sum of A Delta (log2 units) over the chunk's rows (first quarter)
            float d = 0.f, a = 0.f;
            if (qt == 0) {
                if (rvalid) {
                    const float v = dtv + bias;
                    d = p.softplus ? softplus_f(v) : v;
                }
                a = d * A2;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float n = __shfl_up_sync(0xffffffffu, a, o);
                    if (lane >= o) a += n;
                }
                if (lane == 31) wsum[quarter] = a;
            }
            __syncthreads();
            if (qt == 0) {
#pragma unroll
                for (int w = 0; w < 3; ++w)
                    if (w < quarter) a += wsum[w];
                alpha[row] = a;
                dlt[row] = d;
            }

            __syncthreads();  // alpha, delta visible

            const uint32_t sB = sbase + OFF_B + buf * kTile128;
            const uint32_t sX = sbase + OFF_X + buf * kTile64, sM = sbase + OFF_M;
            mma_wait();  // G and Y_off of this chunk, issued when its tiles and the state were ready
            if (!wait_phase(bar_yoff, ph_yoff)) ok = false;
            ph_yoff ^= 1u;
            tc_fence_after();

            // ---- M = G o exp(a_t - a_s) Delta_s [s <= t], bfloat16: row t, columns of this quarter
            {
                const float at = alpha[row];
                const int t = row;
#pragma unroll
                for (int qq = 0; qq < Q / NQ / 32; ++qq) {  // 32 columns at a time
                    const int q = (Q / NQ / 32) * qt + qq;
                    float g[32];
                    tmem_ld32(tmem + tlane + TM_G + q * 32, g);
                    const bool any = q * 32 <= quarter * 32 + 31;  // some row of this warp reaches these columns
#pragma unroll
                    for (int j4 = 0; j4 < 4; ++j4) {  // 8 columns per 16-byte chunk
                        const int sb = q * 32 + j4 * 8;
                        float as[8], ds[8];
                        *reinterpret_cast<float4 *>(as) = *reinterpret_cast<const float4 *>(alpha + sb);  // uniform
                        *reinterpret_cast<float4 *>(as + 4) = *reinterpret_cast<const float4 *>(alpha + sb + 4);
                        *reinterpret_cast<float4 *>(ds) = *reinterpret_cast<const float4 *>(dlt + sb);
                        *reinterpret_cast<float4 *>(ds + 4) = *reinterpret_cast<const float4 *>(dlt + sb + 4);
                        float m[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int s = sb + e;
                            float v = 0.f;
                            if (any && s <= t) v = g[j4 * 8 + e] * ex2_approx(at - as[e]) * ds[e];
                            m[e] = v;
                        }
                        sts128(sM + (sb >> 6) * kTile64 + sw_off(t, (sb & 63) >> 3),
                               make_uint4(pack_bf16(m[0], m[1]), pack_bf16(m[2], m[3]), pack_bf16(m[4], m[5]),
                                          pack_bf16(m[6], m[7])));
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();

            // ---- Y_diag = M X
            if (tid == 0) {
                tc_fence_after();
                constexpr uint32_t iY = idesc_bf16(128, 64, 0, 1);
#pragma unroll
                for (int kk = 0; kk < Q / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * kTile64 + (kk & 3) * 32;
                    umma(tmem + TM_YDIAG, sw128_desc(sM + koff, 16, 1024), sw128_desc(sX + kk * 2048, kTile64, 1024),
                         iY, kk > 0);
                }
                umma_commit(bar_mma);
            }
            mma_wait();

            // ---- x rows scaled in place by w_s = exp(a_Q - a_s) Delta_s: the operand of the state
            // update; the raw row stays in registers for the skip D x of the epilogue (float32: a
            // skip term rounded to bfloat16 inside M would cost up to 2^-9 |D x| where C h and D x
            // nearly cancel)
            const float alast = alpha[Q - 1];
            uint4 xr[PC];
            {
                const int s = row;
                const float w = ex2_approx(alast - alpha[s]) * dlt[s];
#pragma unroll
                for (int j = 0; j < PC; ++j) {
                    const uint32_t ad = sX + sw_off(s, PC * qt + j);
                    const uint4 v = lds128(ad);
                    xr[j] = v;
                    const float2 e0 = unpack_bf16(v.x), e1 = unpack_bf16(v.y), e2 = unpack_bf16(v.z), e3 = unpack_bf16(v.w);
                    sts128(ad, make_uint4(pack_bf16(e0.x * w, e0.y * w), pack_bf16(e1.x * w, e1.y * w),
                                          pack_bf16(e2.x * w, e2.y * w), pack_bf16(e3.x * w, e3.y * w)));
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();

            // ---- S_acc = B^T (w x): A is B read N-major (rows n across the two 64-column blocks)
            if (tid == 0) {
                tc_fence_after();
                constexpr uint32_t iS = idesc_bf16(128, 64, 1, 1);
#pragma unroll
                for (int kk = 0; kk < Q / 16; ++kk)
                    umma(tmem + TM_S, sw128_desc(sB + kk * 2048, kTile64, 1024), sw128_desc(sX + kk * 2048, kTile64, 1024),
                         iS, kk > 0);
                umma_commit(bar_mma);
            }

            // ---- epilogue (overlaps the state MMA): y = Y_diag + exp(a_t) Y_off + D x, gate, store
            {
                const float et = ex2_approx(alpha[row]);
                float yd[PH], yo[PH];
                tmem_ld16(tmem + tlane + TM_YDIAG + qt * PH, yd);
                tmem_ld16(tmem + tlane + TM_YOFF + qt * PH, yo);
                uint32_t out[PH / 2];
#pragma unroll
                for (int e = 0; e < PH; e += 2) {
                    const float2 xx = unpack_bf16((&xr[0].x)[e >> 1]);
                    float v0 = fmaf(dskip, xx.x, fmaf(et, yo[e], yd[e]));
                    float v1 = fmaf(dskip, xx.y, fmaf(et, yo[e + 1], yd[e + 1]));
                    if (p.z) {
                        const float2 zz = unpack_bf16(rvalid ? (&zr[0].x)[e >> 1] : 0u);
                        v0 *= silu_1sfu(zz.x);
                        v1 *= silu_1sfu(zz.y);
                    }
                    out[e >> 1] = pack_bf16(v0, v1);
                }
                if (rvalid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.y + (int64_t(b) * p.L + trow) * (p.H * P) + h * P + qt * PH);
#pragma unroll
                    for (int j = 0; j < PC; ++j) dst[j] = make_uint4(out[4 * j], out[4 * j + 1], out[4 * j + 2], out[4 * j + 3]);
                }
            }
            mma_wait();

            // ---- S <- exp(a_Q) S + S_acc (row n, this quarter's columns), and its bfloat16 parts
            {
                const float eq = ex2_approx(alast);
                float sa[PH];
                tmem_ld16(tmem + tlane + TM_S + qt * PH, sa);
#pragma unroll
                for (int e = 0; e < PH; ++e) S[e] = fmaf(eq, S[e], sa[e]);
            }
            store_S();
            fence_proxy_async_smem();
            tc_fence_before();
            // a wait that gave up ends the block's work (every later wait would give up too)
            const int all_ok = __syncthreads_and(ok);
            tc_fence_after();
            if (!all_ok) break;
            if (c + 1 < c1) issue_G_Yoff(buf ^ 1);
        }
        if (!__syncthreads_and(ok)) break;

        // ---- the segment's end state: published for the next segment, or h_last
        if (k == p.K - 1) {
            if (p.h_last) {
#pragma unroll
                for (int q = 0; q < PH; ++q) p.h_last[((int64_t(b) * p.H + h) * P + PH * qt + q) * NS + row] = S[q];
            }
        } else {
            float4 *dst = reinterpret_cast<float4 *>(p.carry + (bh * NS + row) * P + PH * qt);
#pragma unroll
            for (int q = 0; q < PH / 4; ++q) dst[q] = make_float4(S[4 * q], S[4 * q + 1], S[4 * q + 2], S[4 * q + 3]);
            __threadfence();
            __syncthreads();
            if (tid == 0) st_release_gpu(p.flags + bh, uint32_t(k + 1));
        }
        __syncthreads();
    }
    if (!ok) atomicExch(p.status, uint32_t(SSM_ERR_TIMEOUT));
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace ssd
}  // namespace ssm

// =================================================================== host
namespace {

constexpr size_t kSsdHeader = 256;
inline size_t up256(size_t v) { return (v + 255) / 256 * 256; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// [B, L, inner] bfloat16 as a 3-D map with [64 x 128 x 1] boxes and the 128-byte swizzle.
bool map_sw128(CUtensorMap *m, const void *ptr, int64_t Bsz, int64_t L, int64_t inner) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {cuuint64_t(inner), cuuint64_t(L), cuuint64_t(Bsz)};
    cuuint64_t strides[2] = {cuuint64_t(inner * 2), cuuint64_t(L * inner * 2)};
    cuuint32_t box[3] = {64, cuuint32_t(ssm::ssd::Q), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool al(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t ssd_ws_bytes(int64_t Bsz, int64_t H) {
    if (Bsz <= 0 || H <= 0 || H > (int64_t(1) << 20) || Bsz > (int64_t(1) << 20)) return 0;
    const size_t bh = size_t(Bsz) * size_t(H);
    return up256(kSsdHeader + bh * 4) + bh * ssm::ssd::NS * ssm::ssd::P * 4;
}

ssm_status ssd_validate(const ssm_ssd_args *a) {
    if (!a) return SSM_ERR_INVALID;
    if (a->batch < 0 || a->seqlen < 0 || a->nheads < 0) return SSM_ERR_INVALID;
    if (a->flags & ~uint32_t(SSM_DELTA_SOFTPLUS)) return SSM_ERR_INVALID;
    if (a->dtype != SSM_BF16 || a->headdim != ssm::ssd::P || a->dstate != ssm::ssd::NS) return SSM_ERR_UNSUPPORTED;
    if (a->batch > INT32_MAX || a->seqlen > INT32_MAX || a->nheads > (int64_t(1) << 20)) return SSM_ERR_UNSUPPORTED;
    const bool work = a->batch > 0 && a->nheads > 0 && a->seqlen > 0;
    if (work && (!a->x || !a->dt || !a->Bm || !a->Cm || !a->A || !a->y)) return SSM_ERR_INVALID;
    const void *p16[] = {a->x, a->z, a->y, a->Bm, a->Cm, a->workspace, a->h0, a->h_last};
    for (const void *q : p16)
        if (q && !al(q, 16)) return SSM_ERR_UNSUPPORTED;
    const void *p4[] = {a->A, a->Dskip, a->dt_bias};
    for (const void *q : p4)
        if (q && !al(q, 4)) return SSM_ERR_UNSUPPORTED;
    if (a->dt && !al(a->dt, 2)) return SSM_ERR_UNSUPPORTED;
    if (work && (!a->workspace || a->workspace_bytes < ssd_ws_bytes(a->batch, a->nheads))) return SSM_ERR_INVALID;
    return SSM_OK;
}

}  // namespace

extern "C" {

size_t ssm_ssd_workspace_size(const ssm_ssd_args *a) {
    if (!a) return 0;
    return ssd_ws_bytes(a->batch, a->nheads);
}

ssm_status ssm_ssd_fwd(const ssm_ssd_args *a, void *stream_) {
    using namespace ssm::ssd;
    const ssm_status v = ssd_validate(a);
    if (v != SSM_OK) return v;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (a->batch == 0 || a->nheads == 0) return SSM_OK;
    const size_t hbytes = size_t(a->batch) * size_t(a->nheads) * P * NS * 4;
    if (a->seqlen == 0) {
        if (!a->h_last) return SSM_OK;
        const cudaError_t e = a->h0 ? cudaMemcpyAsync(a->h_last, a->h0, hbytes, cudaMemcpyDeviceToDevice, stream)
                                    : cudaMemsetAsync(a->h_last, 0, hbytes, stream);
        return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
    }
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SSM_ERR_CUDA;
    static std::mutex mu;
    static bool attr_set[64] = {};
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 0 || dev >= 64) return SSM_ERR_CUDA;
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(ssd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_BYTES)) !=
                cudaSuccess)
                return SSM_ERR_CUDA;
            attr_set[dev] = true;
        }
    }
    CUtensorMap tb, tc, tx;
    const int64_t D = a->nheads * P;
    if (!map_sw128(&tb, a->Bm, a->batch, a->seqlen, NS) || !map_sw128(&tc, a->Cm, a->batch, a->seqlen, NS) ||
        !map_sw128(&tx, a->x, a->batch, a->seqlen, D))
        return SSM_ERR_CUDA;
    unsigned char *ws = static_cast<unsigned char *>(a->workspace);
    const int64_t BH = a->batch * a->nheads;
    if (cudaMemsetAsync(ws, 0, kSsdHeader + size_t(BH) * 4, stream) != cudaSuccess) return SSM_ERR_CUDA;
    Params p;
    p.Bsz = a->batch;
    p.L = a->seqlen;
    p.H = a->nheads;
    p.nchunks = (a->seqlen + Q - 1) / Q;
    p.K = (p.nchunks + SEG - 1) / SEG;
    p.items = BH * p.K;
    p.dt = static_cast<const __nv_bfloat16 *>(a->dt);
    p.z = static_cast<const __nv_bfloat16 *>(a->z);
    p.y = static_cast<__nv_bfloat16 *>(a->y);
    p.A = a->A;
    p.Dskip = a->Dskip;
    p.dt_bias = a->dt_bias;
    p.h0 = a->h0;
    p.h_last = a->h_last;
    p.counter = reinterpret_cast<uint32_t *>(ws);
    p.status = reinterpret_cast<uint32_t *>(ws + 4);
    p.flags = reinterpret_cast<uint32_t *>(ws + kSsdHeader);
    p.carry = reinterpret_cast<float *>(ws + up256(kSsdHeader + size_t(BH) * 4));
    p.softplus = (a->flags & SSM_DELTA_SOFTPLUS) != 0;
    const int grid = int(std::min<int64_t>(p.items, sms));
    void *args[] = {&tb, &tc, &tx, &p};
    const cudaError_t e = cudaLaunchKernel(reinterpret_cast<void *>(ssd_kernel), dim3(grid), dim3(NTHREADS), args,
                                           SMEM_BYTES, stream);
    return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // extern "C"
