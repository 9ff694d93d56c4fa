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
// (kind::f16, bfloat16 operands from shared memory, M from tensor memory, float32
// accumulators in tensor memory): G 128x128x128, C [S_hi S_lo] 128x128x128 (S in two
// bfloat16 parts side by side), M X 128x64x128, (w B)^T X 128x64x128.
//
// Work decomposition: one persistent block per SM claims (sequence, head, segment) items in
// order; a segment of SEG chunks starts from the state its predecessor segment published
// (bounded release/acquire wait, as in the scan kernel), so the blocks stay balanced for
// any number of heads.
//
// Within an item the chunks are software-pipelined. Of a chunk's products only C S needs
// the state left by the chunk before; G, M X and B^T (w x) do not. So the products of
// chunk c+1 that do not need the state are issued while chunk c is finished: the sixteen
// compute warps turn chunk c's accumulators into its rows of y and the new state, then
// build chunk c+1's M from its G, while a seventeenth warp issues the TMA loads (two
// chunks ahead) and every MMA as soon as its operands are ready. The weights w of the
// state update scale B's rows in place (after G has read them), so that M X and
// B^T (w x) read the same unscaled x and are issued together.
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
constexpr int NCW = 4 * NQ;          // compute warps; warp w owns tensor-memory lanes (rows) 32 (w mod 4) .. +31
constexpr int NCOMP = 32 * NCW;      // compute threads
constexpr int NTHREADS = NCOMP + 32; // + the load / MMA warp
constexpr int SEG = 16;       // chunks per segment (2048 steps)
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Shared memory (every tile 1024-byte aligned: the 128-byte swizzle repeats every 8 rows).
// A [rows][128 columns] bfloat16 tile is stored as two [rows][64] blocks of 128-byte rows.
constexpr uint32_t kTile128 = Q * 128 * 2;  // 32 KB: [128][128] bf16
constexpr uint32_t kTile64 = Q * 64 * 2;    // 16 KB: [128][64] bf16
constexpr uint32_t OFF_B = 0;                        // B chunk [t][n], two buffers
constexpr uint32_t OFF_C = OFF_B + 2 * kTile128;     // C chunk [t][n], two buffers
constexpr uint32_t OFF_X = OFF_C + 2 * kTile128;     // x chunk [t][p], two buffers
constexpr uint32_t OFF_Z = OFF_X + 2 * kTile64;      // z chunk [t][p] (the gate), one buffer
constexpr uint32_t OFF_S = OFF_Z + kTile64;          // S [n][p] bfloat16, high part (operand of C S)
constexpr uint32_t OFF_SLO = OFF_S + kTile64;        // S - high part, rounded to bfloat16 again
constexpr uint32_t OFF_MISC = OFF_SLO + kTile64;
constexpr uint32_t OFF_ALPHA = OFF_MISC;             // a_t log2 e per row [2][Q] f32, by the chunk's parity
constexpr uint32_t OFF_DELTA = OFF_ALPHA + 2 * Q * 4;  // Delta_t per row [2][Q] f32, by the chunk's parity
constexpr uint32_t OFF_CF = OFF_DELTA + 2 * Q * 4;   // column factors exp(a_r - a_s) Delta_s [2][4][Q] f32, r = 32 rb
constexpr uint32_t OFF_BAR = OFF_CF + 2 * 4 * Q * 4; // mbarriers (12)
constexpr uint32_t OFF_TMEM = OFF_BAR + 128;         // tensor-memory base address
constexpr uint32_t OFF_ITEM = OFF_TMEM + 16;         // claimed item, abort flag
constexpr uint32_t SMEM_BYTES = OFF_ITEM + 16 + 1024;  // + slack to align the base to 1024
static_assert(SMEM_BYTES <= 232448, "227 KB of shared memory per block");
constexpr uint32_t kLoadBytes = 2 * kTile128 + kTile64;  // one chunk: B, C, x

// Tensor memory: 512 columns x 128 lanes of 32 bits: G [128 cols], M X [64], B^T (w x) [64],
// C S as [C S_hi | C S_lo] [128], and M itself [64: two bfloat16 per column], the A operand of
// M X read by the tensor cores from tensor memory.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t TM_G = 0, TM_YDIAG = 128, TM_S = 192, TM_YOFF = 256, TM_M = 384;

struct Params {
    int64_t Bsz, L, H, nchunks, K, items;  // K: segments per sequence
    const __nv_bfloat16 *dt, *z;
    __nv_bfloat16 *y;
    const float *A, *Dskip, *dt_bias, *h0;
    float *h_last;
    uint32_t *counter, *status, *flags;
    float *carry;  // [B*H][NS][P]
    int softplus, drop_handoff;
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
// The same with A read from tensor memory (a_tmem: its first column; K = 16 bfloat16 in 8 columns).
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
// 8 consecutive 32-bit columns of this thread's lane written (32x32b shape); then the wait.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
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

// Bounded wait on phase `parity` of an mbarrier. A wait that gives up sets the block's abort
// flag, and every wait returns false at once while it is set, so that a block whose
// hand-offs broke runs through its remaining steps without waiting and stops at the next item.
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort) return false;
        if (globaltimer_ns() - start > kWaitLimitNs) {
            *abort = 1;
            return false;
        }
    }
    return true;
}
__device__ __forceinline__ void mbar_arrive1(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Barrier of the compute warps alone (named barrier 1).
__device__ __forceinline__ void comp_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NCOMP) : "memory"); }

// 16 float32 columns of this thread's lane without waiting, and the wait that makes them
// valid (the registers pass through it, so no use can move above it).
__device__ __forceinline__ void tmem_ld16_nw(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld8_nw(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_wait8(uint32_t (&r)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_wait16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
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
               const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z, const Params p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    float *alpha = reinterpret_cast<float *>(smem + OFF_ALPHA);
    float *dlt = reinterpret_cast<float *>(smem + OFF_DELTA);
    float *cfac = reinterpret_cast<float *>(smem + OFF_CF);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *bar_full = bars;    // [2] a chunk's B, C and x tiles have landed (TMA)
    uint64_t *bar_g = bars + 2;   // G done
    uint64_t *bar_yd = bars + 3;  // M X done
    uint64_t *bar_sa = bars + 10; // B^T (w x) done
    uint64_t *bar_br = bars + 11; // the compute threads: B scaled
    uint64_t *bar_yo = bars + 4;  // C S done
    uint64_t *bar_sr = bars + 5;  // the compute threads: state stored, the chunk's accumulators, x and z read
    uint64_t *bar_mr = bars + 6;  // the compute threads: M written, G read
    uint64_t *bar_pf = bars + 7;  // [2] the load warp: a chunk's Delta and prefix stored (by the chunk's parity)
    uint64_t *bar_z = bars + 9;   // z of the next chunk to finish has landed (TMA)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_TMEM);
    int *item_slot = reinterpret_cast<int *>(smem + OFF_ITEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_ITEM + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Compute threads: row (tensor-memory lane) and column quarter qt; warps w, w+4, w+8, w+12
    // share the lanes 32 (w mod 4) .. +31, warp w + 4 qt taking quarter qt of every row.
    const int row = tid & (Q - 1), qt = tid >> 7, quarter = warp & 3;
    const bool gate = p.z != nullptr;

    if (tid == 0) {
        mbar_init(&bar_full[0], 1);
        mbar_init(&bar_full[1], 1);
        mbar_init(bar_g, 1);
        mbar_init(bar_yd, 1);
        mbar_init(bar_sa, 1);
        mbar_init(bar_br, NCOMP);
        mbar_init(bar_yo, 1);
        mbar_init(bar_sr, NCOMP);
        mbar_init(bar_mr, NCOMP);
        mbar_init(&bar_pf[0], 32);
        mbar_init(&bar_pf[1], 32);
        mbar_init(bar_z, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_b);
        prefetch_tensormap(&tm_c);
        prefetch_tensormap(&tm_x);
        if (gate) prefetch_tensormap(&tm_z);
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
    // mbarrier phases, carried across items (each role uses its own)
    uint32_t ph_full0 = 0, ph_full1 = 0, ph_g = 0, ph_yd = 0, ph_sa = 0, ph_br = 0, ph_yo = 0, ph_sr = 0;
    uint32_t ph_mr = 0, ph_pf0 = 0, ph_pf1 = 0, ph_z = 0;
    auto wait_bar = [&](uint64_t *bar, uint32_t &ph) {
        wait_phase(bar, ph, abort_flag);
        ph ^= 1u;
        tc_fence_after();
    };

    for (;;) {
        if (tid == 0) *item_slot = int(atomicAdd(p.counter, 1u));
        __syncthreads();
        const int64_t it = *item_slot;
        if (it >= p.items || *abort_flag) break;
        const int64_t bh = it % (p.Bsz * p.H), k = it / (p.Bsz * p.H);
        const int b = int(bh / p.H), h = int(bh % p.H);
        const int64_t c0 = k * SEG, c1 = c0 + SEG < p.nchunks ? c0 + SEG : p.nchunks;
        const int nch = int(c1 - c0);
        const float A2 = __ldg(p.A + h) * kLog2e;  // A log2 e

        if (warp == NCW) {
            // ---------------- load / MMA warp: lane 0 issues, every lane waits
            const bool lead = lane == 0;
            const float bias = p.dt_bias ? __ldg(p.dt_bias + h) : 0.f;
            auto issue_loads = [&](int64_t c, int buf) {  // B and C as two 64-column boxes each, x one
                if (!lead || *abort_flag) return;
                const int t0 = int(c * Q);
                mbar_arrive_expect_tx(&bar_full[buf], kLoadBytes);
                unsigned char *bb = smem + OFF_B + buf * kTile128, *cc = smem + OFF_C + buf * kTile128;
                tma_load_3d(bb, &tm_b, &bar_full[buf], 0, t0, b);
                tma_load_3d(bb + kTile64, &tm_b, &bar_full[buf], 64, t0, b);
                tma_load_3d(cc, &tm_c, &bar_full[buf], 0, t0, b);
                tma_load_3d(cc + kTile64, &tm_c, &bar_full[buf], 64, t0, b);
                tma_load_3d(smem + OFF_X + buf * kTile64, &tm_x, &bar_full[buf], h * P, t0, b);
            };
            auto issue_z = [&](int64_t c) {
                if (!gate || !lead || *abort_flag) return;
                mbar_arrive_expect_tx(bar_z, kTile64);
                tma_load_3d(smem + OFF_Z, &tm_z, bar_z, h * P, int(c * Q), b);
            };
            // G = C B^T of the chunk in buffer buf, once its tiles have landed
            auto issue_G = [&](int buf) {
                uint32_t &ph = buf ? ph_full1 : ph_full0;
                wait_phase(&bar_full[buf], ph, abort_flag);
                ph ^= 1u;
                tc_fence_after();
                if (!lead || *abort_flag) return;
                const uint32_t sB = sbase + OFF_B + buf * kTile128, sC = sbase + OFF_C + buf * kTile128;
                constexpr uint32_t iG = idesc_bf16(128, 128, 0, 0);
#pragma unroll
                for (int kk = 0; kk < NS / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * kTile64 + (kk & 3) * 32;  // K block, 32 bytes per 16 columns
                    umma(tmem + TM_G, sw128_desc(sC + koff, 16, 1024), sw128_desc(sB + koff, 16, 1024), iG, kk > 0);
                }
                umma_commit(bar_g);
            };
            // C [S_hi | S_lo]: one N = 128 product (S_lo's block follows S_hi's, 16 KB on)
            auto issue_Yoff = [&](int buf) {
                if (!lead || *abort_flag) return;
                const uint32_t sC = sbase + OFF_C + buf * kTile128;
                constexpr uint32_t iO = idesc_bf16(128, 128, 0, 1);
#pragma unroll
                for (int kk = 0; kk < NS / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * kTile64 + (kk & 3) * 32;
                    umma(tmem + TM_YOFF, sw128_desc(sC + koff, 16, 1024), sw128_desc(sbase + OFF_S + kk * 2048, kTile64, 1024),
                         iO, kk > 0);
                }
                umma_commit(bar_yo);
            };
            // M X (M from tensor memory), as soon as M is written; then (w B)^T x, once B's rows
            // are scaled: both read the chunk's unscaled x, each has its own completion
            auto issue_Yd = [&](int buf) {
                if (!lead || *abort_flag) return;
                const uint32_t sX = sbase + OFF_X + buf * kTile64;
                constexpr uint32_t iY = idesc_bf16(128, 64, 0, 1);
#pragma unroll
                for (int kk = 0; kk < Q / 16; ++kk)
                    umma_ts(tmem + TM_YDIAG, tmem + TM_M + kk * 8, sw128_desc(sX + kk * 2048, kTile64, 1024), iY, kk > 0);
                umma_commit(bar_yd);
            };
            auto issue_Sa = [&](int buf) {
                if (!lead || *abort_flag) return;
                const uint32_t sB = sbase + OFF_B + buf * kTile128, sX = sbase + OFF_X + buf * kTile64;
                constexpr uint32_t iS = idesc_bf16(128, 64, 1, 1);  // A is B read N-major (rows n across its two blocks)
#pragma unroll
                for (int kk = 0; kk < Q / 16; ++kk)
                    umma(tmem + TM_S, sw128_desc(sB + kk * 2048, kTile64, 1024), sw128_desc(sX + kk * 2048, kTile64, 1024),
                         iS, kk > 0);
                umma_commit(bar_sa);
            };
            // dt of the chunk's rows 4 lane .. 4 lane + 3 (rows past L read row L - 1; the prefix
            // zeroes them), loaded a loader iteration before its use: the raw bits ride in registers
            // over the loop's back edge and are widened only there
            auto load_dt4 = [&](int64_t c, uint16_t (&v)[4]) {  // raw bits: widened where used, so no wait here
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int64_t t = c * Q + 4 * lane + j;
                    v[j] = ldg_u16_early(p.dt + (int64_t(b) * p.L + (t < p.L ? t : p.L - 1)) * p.H + h);
                }
            };
            // Delta_t and a_t = A (Delta_1 + ... + Delta_t) log2 e of chunk c (slot = its parity in the
            // item) from its dt: lane l takes rows 4l .. 4l+3, a running sum over them, then a scan of
            // the lanes' totals; every lane arrives once its rows are stored
            auto prefix = [&](int64_t c, int slot, const uint16_t (&dtv)[4]) {
                float d4[4], a4[4];
                float run = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int64_t t = c * Q + 4 * lane + j;
                    float d = 0.f;
                    if (t < p.L) {
                        const float v = __uint_as_float(uint32_t(dtv[j]) << 16) + bias;
                        d = p.softplus ? softplus_f(v) : v;
                    }
                    d4[j] = d;
                    run = fmaf(d, A2, run);
                    a4[j] = run;
                }
                float excl = run;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float n = __shfl_up_sync(0xffffffffu, excl, o);
                    if (lane >= o) excl += n;
                }
                excl -= run;  // sum of the preceding lanes' rows
                *reinterpret_cast<float4 *>(alpha + slot * Q + 4 * lane) =
                    make_float4(a4[0] + excl, a4[1] + excl, a4[2] + excl, a4[3] + excl);
                *reinterpret_cast<float4 *>(dlt + slot * Q + 4 * lane) = make_float4(d4[0], d4[1], d4[2], d4[3]);
                // the factors exp(a_r - a_s) Delta_s of the columns s < r = 32 rb wholly left of row
                // block rb (a_r - a_s <= 0: at most 1); the other columns' entries are not read
#pragma unroll
                for (int rb = 1; rb < 4; ++rb) {
                    const float ar = __shfl_sync(0xffffffffu, a4[0] + excl, 8 * rb);  // row 32 rb is lane 8 rb's first
                    float cfv[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        cfv[j] = 4 * lane + j < 32 * rb ? ex2_approx(ar - (a4[j] + excl)) * d4[j] : 0.f;
                    *reinterpret_cast<float4 *>(cfac + (slot * 4 + rb) * Q + 4 * lane) = make_float4(cfv[0], cfv[1], cfv[2], cfv[3]);
                }
                mbar_arrive1(&bar_pf[slot]);
            };

            uint16_t dta[4], dtb[4];
            load_dt4(c0, dta);
            load_dt4(c0 + 1, dtb);
            issue_loads(c0, 0);
            if (nch > 1) issue_loads(c0 + 1, 1);
            issue_z(c0);
            prefix(c0, 0, dta);
            issue_G(0);
            wait_bar(bar_sr, ph_sr);  // the segment's start state is in shared memory
            issue_Yoff(0);
            if (nch > 1) prefix(c0 + 1, 1, dtb);
            load_dt4(c0 + 2, dta);
            wait_bar(bar_mr, ph_mr);  // chunk c0's M
            issue_Yd(0);
            wait_bar(bar_br, ph_br);  // chunk c0's B scaled
            issue_Sa(0);
            if (nch > 1) issue_G(1);
            for (int i = 0; i < nch; ++i) {
                wait_bar(bar_sr, ph_sr);  // chunk c0+i finished: its buffer and z's are free, the new state stored
                if (i + 2 < nch) issue_loads(c0 + i + 2, i & 1);
                if (i + 1 < nch) {
                    issue_z(c0 + i + 1);
                    issue_Yoff((i + 1) & 1);
                    wait_bar(bar_mr, ph_mr);  // chunk c0+i+1's M
                    issue_Yd((i + 1) & 1);
                    wait_bar(bar_br, ph_br);  // chunk c0+i+1's B scaled
                    issue_Sa((i + 1) & 1);
                    if (i + 2 < nch) {
                        issue_G(i & 1);
                        prefix(c0 + i + 2, i & 1, dta);
                        load_dt4(c0 + i + 3, dta);
                    }
                }
            }
            __syncwarp();
        } else {
            // ---------------- compute warps
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
                comp_sync();
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
            // bfloat16 parts, S = hi + lo to about 2^-17, so that C S keeps the float32 state's
            // precision; then the hand-off to the MMA warp (every thread fences its stores for
            // the tensor cores and orders its tensor-memory reads before arriving)
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
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive1(bar_sr);
            };
            store_S();

            // M = G o exp(a_t - a_s) Delta_s [s <= t] (bfloat16 pairs, row t, this quarter's 32
            // columns) into tensor memory, and B's row s scaled in place by w_s = exp(a_Q - a_s)
            // Delta_s (this quarter's 32 columns; G has read B); then the hand-off
            auto build_M = [&](int slot) {
                wait_bar(&bar_pf[slot], slot ? ph_pf1 : ph_pf0);
                wait_bar(bar_g, ph_g);
                const float *al = alpha + slot * Q, *dl = dlt + slot * Q;
                const float at = al[row];
                const int t = row;
                // columns wholly left of this warp's row block r = 32 quarter: exp(a_t - a_s) =
                // exp(a_t - a_r) exp(a_r - a_s), the second factor (times Delta_s) per column
                const float rt = quarter ? ex2_approx(at - al[32 * quarter]) : 1.f;
                const float *cf = cfac + (slot * 4 + quarter) * Q;
#pragma unroll
                for (int qq = 0; qq < Q / NQ / 16; ++qq) {  // 16 columns at a time
                    const int q = (Q / NQ / 16) * qt + qq;
                    float g[16];
                    tmem_ld16(tmem + tlane + TM_G + q * 16, g);
                    const bool any = q * 16 <= quarter * 32 + 31;  // some row of this warp reaches these columns
                    const bool left = q * 16 + 15 < quarter * 32;  // every row of this warp is past these columns
                    uint32_t mp[8];
#pragma unroll
                    for (int j4 = 0; j4 < 2; ++j4) {  // 8 columns at a time
                        const int sb = q * 16 + j4 * 8;
                        if (left) {
                            float cs[8];
                            *reinterpret_cast<float4 *>(cs) = *reinterpret_cast<const float4 *>(cf + sb);  // uniform
                            *reinterpret_cast<float4 *>(cs + 4) = *reinterpret_cast<const float4 *>(cf + sb + 4);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                mp[j4 * 4 + e] = pack_bf16(g[j4 * 8 + 2 * e] * rt * cs[2 * e], g[j4 * 8 + 2 * e + 1] * rt * cs[2 * e + 1]);
                            continue;
                        }
                        float as[8], ds[8];
                        *reinterpret_cast<float4 *>(as) = *reinterpret_cast<const float4 *>(al + sb);  // uniform
                        *reinterpret_cast<float4 *>(as + 4) = *reinterpret_cast<const float4 *>(al + sb + 4);
                        *reinterpret_cast<float4 *>(ds) = *reinterpret_cast<const float4 *>(dl + sb);
                        *reinterpret_cast<float4 *>(ds + 4) = *reinterpret_cast<const float4 *>(dl + sb + 4);
                        float m[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int s = sb + e;
                            float v = 0.f;
                            if (any && s <= t) v = g[j4 * 8 + e] * ex2_approx(at - as[e]) * ds[e];
                            m[e] = v;
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) mp[j4 * 4 + e] = pack_bf16(m[2 * e], m[2 * e + 1]);
                    }
                    tmem_st8(tmem + tlane + TM_M + q * 8, mp);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive1(bar_mr);  // M X can start
                const float w = ex2_approx(al[Q - 1] - at) * dl[row];
                constexpr int BC = NS / NQ;  // B columns of this thread's part of row s
                const uint32_t sBq = sbase + OFF_B + slot * kTile128 + (qt * BC / 64) * kTile64;
#pragma unroll
                for (int j = 0; j < BC / 8; ++j) {
                    const uint32_t ad = sBq + sw_off(row, (qt * BC % 64) / 8 + j);
                    const uint4 v = lds128(ad);
                    const float2 e0 = unpack_bf16(v.x), e1 = unpack_bf16(v.y), e2 = unpack_bf16(v.z), e3 = unpack_bf16(v.w);
                    sts128(ad, make_uint4(pack_bf16(e0.x * w, e0.y * w), pack_bf16(e1.x * w, e1.y * w),
                                          pack_bf16(e2.x * w, e2.y * w), pack_bf16(e3.x * w, e3.y * w)));
                }
                fence_proxy_async_smem();
                mbar_arrive1(bar_br);
            };
            build_M(0);

            for (int i = 0; i < nch; ++i) {
                const int64_t c = c0 + i;
                const int slot = i & 1;
                const int64_t trow = c * Q + row;
                const bool rvalid = trow < p.L;

                // ---- y = M X + exp(a_t) C S + D x, gate, store (this row, this quarter)
                // first the parts that do not need M X: pre = D x + exp(a_t) C S and the gate
                // silu(z) of the thread's 16 columns, while M X may still be running
                wait_bar(bar_yo, ph_yo);
                if (gate) wait_bar(bar_z, ph_z);
                float pre[PH], gz[PH];
                {
                    const float et = ex2_approx(alpha[slot * Q + row]);
#pragma unroll
                    for (int j = 0; j < PC; ++j) {  // 8 columns at a time
                        uint32_t rh[8], rl[8];
                        tmem_ld8_nw(tmem + tlane + TM_YOFF + qt * PH + 8 * j, rh);
                        tmem_ld8_nw(tmem + tlane + TM_YOFF + P + qt * PH + 8 * j, rl);
                        const uint4 xv = lds128(sbase + OFF_X + slot * kTile64 + sw_off(row, PC * qt + j));
                        const uint4 zv = gate ? lds128(sbase + OFF_Z + sw_off(row, PC * qt + j)) : make_uint4(0, 0, 0, 0);
                        tmem_wait8(rh);
                        tmem_wait8(rl);
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const float2 xx = unpack_bf16((&xv.x)[e >> 1]);
                            const float yo0 = __uint_as_float(rh[e]) + __uint_as_float(rl[e]);
                            const float yo1 = __uint_as_float(rh[e + 1]) + __uint_as_float(rl[e + 1]);
                            pre[8 * j + e] = fmaf(dskip, xx.x, et * yo0);
                            pre[8 * j + e + 1] = fmaf(dskip, xx.y, et * yo1);
                            const float2 zz = unpack_bf16((&zv.x)[e >> 1]);
                            gz[8 * j + e] = gate ? silu_f(zz.x) : 1.f;
                            gz[8 * j + e + 1] = gate ? silu_f(zz.y) : 1.f;
                        }
                    }
                }
                // then y = (M X + pre) silu(z), stored
                wait_bar(bar_yd, ph_yd);
                {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.y + (int64_t(b) * p.L + trow) * (p.H * P) + h * P + qt * PH);
#pragma unroll
                    for (int j = 0; j < PC; ++j) {
                        uint32_t rd[8];
                        tmem_ld8_nw(tmem + tlane + TM_YDIAG + qt * PH + 8 * j, rd);
                        tmem_wait8(rd);
                        uint32_t out[4];
#pragma unroll
                        for (int e = 0; e < 8; e += 2)
                            out[e >> 1] = pack_bf16((__uint_as_float(rd[e]) + pre[8 * j + e]) * gz[8 * j + e],
                                                    (__uint_as_float(rd[e + 1]) + pre[8 * j + e + 1]) * gz[8 * j + e + 1]);
                        if (rvalid) dst[j] = make_uint4(out[0], out[1], out[2], out[3]);
                    }
                }

                // ---- S <- exp(a_Q) S + B^T (w x) (row n, this quarter's columns), stored for C S
                {
                    const float eq = ex2_approx(alpha[slot * Q + Q - 1]);
                    wait_bar(bar_sa, ph_sa);
#pragma unroll
                    for (int k16 = 0; k16 < PH / 16; ++k16) {
                        uint32_t rs[16];
                        tmem_ld16_nw(tmem + tlane + TM_S + qt * PH + 16 * k16, rs);
                        tmem_wait16(rs);
#pragma unroll
                        for (int e = 0; e < 16; ++e) S[16 * k16 + e] = fmaf(eq, S[16 * k16 + e], __uint_as_float(rs[e]));
                    }
                }
                store_S();
                if (i + 1 < nch) build_M(slot ^ 1);
            }

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
                comp_sync();
                // (test hook: the first segment of sequence 0, head 0 keeps its state to itself)
                if (tid == 0 && !(p.drop_handoff && bh == 0 && k == 0)) st_release_gpu(p.flags + bh, uint32_t(k + 1));
            }
        }
        __syncthreads();
    }
    if (tid == 0 && *abort_flag) atomicExch(p.status, uint32_t(SSM_ERR_TIMEOUT));
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
    if (a->flags & ~uint32_t(SSM_DELTA_SOFTPLUS | SSM_TEST_DROP_HANDOFF)) return SSM_ERR_INVALID;
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
    CUtensorMap tb, tc, tx, tz;
    const int64_t D = a->nheads * P;
    if (!map_sw128(&tb, a->Bm, a->batch, a->seqlen, NS) || !map_sw128(&tc, a->Cm, a->batch, a->seqlen, NS) ||
        !map_sw128(&tx, a->x, a->batch, a->seqlen, D) || !map_sw128(&tz, a->z ? a->z : a->x, a->batch, a->seqlen, D))
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
    p.drop_handoff = (a->flags & SSM_TEST_DROP_HANDOFF) != 0;
    const int grid = int(std::min<int64_t>(p.items, sms));
    void *args[] = {&tb, &tc, &tx, &tz, &p};
    const cudaError_t e = cudaLaunchKernel(reinterpret_cast<void *>(ssd_kernel), dim3(grid), dim3(NTHREADS), args,
                                           SMEM_BYTES, stream);
    return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

}  // extern "C"
