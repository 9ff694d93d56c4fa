// ssm_host.cu -- the scan over host-resident tokens: chunked, with host<->device copies
// on two copy streams overlapping each other and the scan kernels (ssm_scan_fwd_host).
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "../../include/ssm_scan.h"

namespace {

inline size_t up256(size_t v) { return (v + 255) / 256 * 256; }

// Staging layout for chunks of Lc steps: two buffers, each x | dt | z | y (B x Lc x D
// tokens), B | C (B x Lc x N tokens) and, with the short convolution, the three tokens
// before the chunk (B x 3 x D); then two carried states [B, D, N] float32.
struct Staging {
    size_t tok, bc, x0, buf, carry, total;
    size_t off_x, off_dt, off_z, off_y, off_b, off_c, off_x0, off_carry;
};

Staging staging_layout(const ssm_scan_args *a, int64_t Lc) {
    Staging s{};
    const size_t es = a->dtype == SSM_BF16 ? 2 : 4;
    s.tok = up256(size_t(a->batch) * size_t(Lc) * size_t(a->dim) * es);
    s.bc = up256(size_t(a->batch) * size_t(Lc) * size_t(a->dstate) * es);
    s.off_x = 0;
    s.off_dt = s.tok;
    s.off_z = 2 * s.tok;
    s.off_y = 3 * s.tok;
    s.off_b = 4 * s.tok;
    s.off_c = 4 * s.tok + s.bc;
    s.x0 = a->conv_w ? up256(size_t(a->batch) * 3 * size_t(a->dim) * es) : 0;
    s.off_x0 = 4 * s.tok + 2 * s.bc;
    s.buf = 4 * s.tok + 2 * s.bc + s.x0;
    s.carry = up256(size_t(a->batch) * size_t(a->dim) * size_t(a->dstate) * 4);
    s.off_carry = 2 * s.buf;
    s.total = 2 * s.buf + 2 * s.carry;
    return s;
}

// Copy streams and events of one device, created on first use and kept.
struct CopyEngine {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t ev_start = nullptr, ev_end = nullptr, ev_in[2] = {}, ev_scan[2] = {}, ev_out[2] = {};
    bool ok = false;
};

constexpr int kMaxDevices = 64;
std::mutex g_mu;  // guards the engines and serialises enqueueing (events are shared)
CopyEngine g_engine[kMaxDevices];

bool engine_init(CopyEngine &e) {
    if (e.ok) return true;
    const unsigned fl = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&e.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&e.out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&e.ev_start, fl) != cudaSuccess || cudaEventCreateWithFlags(&e.ev_end, fl) != cudaSuccess)
        return false;
    for (int i = 0; i < 2; ++i)
        if (cudaEventCreateWithFlags(&e.ev_in[i], fl) != cudaSuccess ||
            cudaEventCreateWithFlags(&e.ev_scan[i], fl) != cudaSuccess ||
            cudaEventCreateWithFlags(&e.ev_out[i], fl) != cudaSuccess)
            return false;
    e.ok = true;
    return true;
}

// Rows [t0, t0 + n) of a [B, L, inner] tensor between host and a contiguous [B, n, inner]
// device buffer: one strided copy (B rows of n * inner elements).
cudaError_t copy_rows(void *dst, const void *src, const ssm_scan_args *a, int64_t inner, int64_t t0, int64_t n,
                      bool to_device, cudaStream_t st) {
    const size_t es = a->dtype == SSM_BF16 ? 2 : 4;
    const size_t width = size_t(n) * size_t(inner) * es, host_pitch = size_t(a->seqlen) * size_t(inner) * es;
    const size_t host_off = size_t(t0) * size_t(inner) * es;
    if (to_device)
        return cudaMemcpy2DAsync(dst, width, static_cast<const unsigned char *>(src) + host_off, host_pitch, width,
                                 size_t(a->batch), cudaMemcpyHostToDevice, st);
    return cudaMemcpy2DAsync(static_cast<unsigned char *>(dst) + host_off, host_pitch, src, width, width,
                             size_t(a->batch), cudaMemcpyDeviceToHost, st);
}

// The three tokens before step t0 ([B, 3, D], oldest first), the short convolution's
// prefix for a chunk that starts at t0 > 0: rows t0-3 .. t0-1 of the host x, and before
// t = 0 the caller's device prefix (or zeros).
cudaError_t copy_prefix(void *dst, const ssm_scan_args *a, int64_t t0, cudaStream_t st) {
    const size_t es = a->dtype == SSM_BF16 ? 2 : 4;
    const size_t row = size_t(a->dim) * es, pitch = 3 * row, host_pitch = size_t(a->seqlen) * row;
    const unsigned char *x = static_cast<const unsigned char *>(a->x);
    if (t0 >= 3)
        return cudaMemcpy2DAsync(dst, pitch, x + size_t(t0 - 3) * row, host_pitch, pitch, size_t(a->batch),
                                 cudaMemcpyHostToDevice, st);
    for (int r = 0; r < 3; ++r) {  // chunks shorter than three steps
        unsigned char *d = static_cast<unsigned char *>(dst) + r * row;
        const int64_t tau = t0 - 3 + r;
        cudaError_t e;
        if (tau >= 0)
            e = cudaMemcpy2DAsync(d, pitch, x + size_t(tau) * row, host_pitch, row, size_t(a->batch),
                                  cudaMemcpyHostToDevice, st);
        else if (a->conv_x0)
            e = cudaMemcpy2DAsync(d, pitch, static_cast<const unsigned char *>(a->conv_x0) + size_t(tau + 3) * row,
                                  pitch, row, size_t(a->batch), cudaMemcpyDeviceToDevice, st);
        else
            e = cudaMemset2DAsync(d, pitch, 0, row, size_t(a->batch), st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t ssm_scan_host_staging_size(const ssm_scan_args *a, int64_t chunk_len) {
    if (!a || chunk_len < 1 || a->batch < 0 || a->seqlen < 0 || a->dim < 0 || a->dstate < 1) return 0;
    const int64_t Lc = std::min<int64_t>(chunk_len, std::max<int64_t>(a->seqlen, 1));
    return staging_layout(a, Lc).total;
}

ssm_status ssm_scan_fwd_host(const ssm_scan_args *a, int64_t chunk_len, void *staging, size_t staging_bytes,
                             void *stream_) {
    if (!a || chunk_len < 1 || !staging) return SSM_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(staging) & 255) != 0) return SSM_ERR_UNSUPPORTED;
    const size_t need = ssm_scan_host_staging_size(a, chunk_len);
    if (need == 0 || staging_bytes < need) return SSM_ERR_INVALID;
    if (a->batch == 0 || a->dim == 0) return SSM_OK;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (a->seqlen == 0) return ssm_scan_fwd(a, stream);  // no tokens to move: only h_last
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    CopyEngine &e = g_engine[dev];
    if (!engine_init(e)) return SSM_ERR_CUDA;

    const int64_t Lc = std::min<int64_t>(chunk_len, a->seqlen);
    const Staging s = staging_layout(a, Lc);
    unsigned char *base = static_cast<unsigned char *>(staging);
    float *carry[2] = {reinterpret_cast<float *>(base + s.off_carry),
                       reinterpret_cast<float *>(base + s.off_carry + s.carry)};
    const int64_t nc = (a->seqlen + Lc - 1) / Lc;
    // On an error after copies were queued, wait for both copy streams before returning,
    // so that the caller may reuse or free its page-locked buffers at once.
    auto fail = [&](ssm_status st) {
        cudaStreamSynchronize(e.in);
        cudaStreamSynchronize(e.out);
        return st;
    };
#define SSM_CK(call)                                          \
    do {                                                      \
        if ((call) != cudaSuccess) return fail(SSM_ERR_CUDA); \
    } while (0)
    // Everything starts after the work already on `stream` (it may still use the staging memory).
    SSM_CK(cudaEventRecord(e.ev_start, stream));
    SSM_CK(cudaStreamWaitEvent(e.in, e.ev_start, 0));
    SSM_CK(cudaStreamWaitEvent(e.out, e.ev_start, 0));
    for (int64_t c = 0; c < nc; ++c) {
        const int k = int(c & 1);
        unsigned char *buf = base + size_t(k) * s.buf;
        const int64_t t0 = c * Lc, n = std::min<int64_t>(Lc, a->seqlen - t0);
        // Copy in chunk c once the scan of chunk c-2 has finished reading this buffer.
        if (c >= 2) SSM_CK(cudaStreamWaitEvent(e.in, e.ev_scan[k], 0));
        SSM_CK(copy_rows(buf + s.off_x, a->x, a, a->dim, t0, n, true, e.in));
        SSM_CK(copy_rows(buf + s.off_dt, a->dt, a, a->dim, t0, n, true, e.in));
        if (a->z) SSM_CK(copy_rows(buf + s.off_z, a->z, a, a->dim, t0, n, true, e.in));
        SSM_CK(copy_rows(buf + s.off_b, a->Bm, a, a->dstate, t0, n, true, e.in));
        SSM_CK(copy_rows(buf + s.off_c, a->Cm, a, a->dstate, t0, n, true, e.in));
        if (a->conv_w && c > 0) SSM_CK(copy_prefix(buf + s.off_x0, a, t0, e.in));
        SSM_CK(cudaEventRecord(e.ev_in[k], e.in));
        // Scan chunk c once its inputs are in and the y of chunk c-2 has left this buffer.
        SSM_CK(cudaStreamWaitEvent(stream, e.ev_in[k], 0));
        if (c >= 2) SSM_CK(cudaStreamWaitEvent(stream, e.ev_out[k], 0));
        ssm_scan_args b = *a;
        b.seqlen = n;
        b.x = buf + s.off_x;
        b.dt = buf + s.off_dt;
        b.z = a->z ? buf + s.off_z : nullptr;
        b.Bm = buf + s.off_b;
        b.Cm = buf + s.off_c;
        b.y = buf + s.off_y;
        b.h0 = c == 0 ? a->h0 : carry[(c - 1) & 1];
        b.h_last = c == nc - 1 ? a->h_last : carry[c & 1];
        if (a->conv_w) b.conv_x0 = c == 0 ? a->conv_x0 : buf + s.off_x0;
        const ssm_status st = ssm_scan_fwd(&b, stream);
        if (st != SSM_OK) return fail(st);
        SSM_CK(cudaEventRecord(e.ev_scan[k], stream));
        // Copy out the y of chunk c.
        SSM_CK(cudaStreamWaitEvent(e.out, e.ev_scan[k], 0));
        SSM_CK(copy_rows(a->y, buf + s.off_y, a, a->dim, t0, n, false, e.out));
        SSM_CK(cudaEventRecord(e.ev_out[k], e.out));
    }
    // Later work on `stream` runs after the last copy out.
    SSM_CK(cudaEventRecord(e.ev_end, e.out));
    SSM_CK(cudaStreamWaitEvent(stream, e.ev_end, 0));
#undef SSM_CK
    return SSM_OK;
}

}  // extern "C"
