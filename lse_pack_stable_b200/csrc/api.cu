// C-ABI entry points of libcplse: host-side validation, then one launch on the
// caller's stream. Contracts are documented in include/cplse.h.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include "cplse.h"
#include "launch.h"

namespace cplse {

int sm_count()
{
    constexpr int kCachedDevices = 64;
    static std::atomic<int> cache[kCachedDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;   // B200; the launch reports the error
    const bool cached = dev >= 0 && dev < kCachedDevices;
    if (cached) {
        const int n = cache[dev].load(std::memory_order_relaxed);
        if (n > 0) return n;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (cached) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace cplse

namespace {

thread_local char g_err[512] = "";

cp_status fail(cp_status st, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

cp_status ok()
{
    g_err[0] = '\0';
    return CP_OK;
}

// The pointer must be device (or managed) memory of the current device.
cp_status check_device_ptr(const void* p, const char* name)
{
    if (p == nullptr) return fail(CP_ERR_ARG, "%s is NULL", name);
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(CP_ERR_ARG, "%s: cudaPointerGetAttributes failed (%s)", name,
                    cudaGetErrorString(e));
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
        return fail(CP_ERR_ARG, "%s is not device memory", name);
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return fail(CP_ERR_CUDA, "cudaGetDevice failed");
    }
    if (at.type == cudaMemoryTypeDevice && at.device != dev)
        return fail(CP_ERR_ARG, "%s lives on device %d, current device is %d", name, at.device,
                    dev);
    return CP_OK;
}

// The pointer must be device memory that the current device can address: its
// own, or another device's (a peer mapping) when the two have peer access.
cp_status check_addressable_ptr(const void* p, const char* name)
{
    if (p == nullptr) return fail(CP_ERR_ARG, "%s is NULL", name);
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(CP_ERR_ARG, "%s: cudaPointerGetAttributes failed (%s)", name,
                    cudaGetErrorString(e));
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
        return fail(CP_ERR_ARG, "%s is not device memory", name);
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return fail(CP_ERR_CUDA, "cudaGetDevice failed");
    }
    if (at.type == cudaMemoryTypeDevice && at.device != dev) {
        int can = 0;
        if (cudaDeviceCanAccessPeer(&can, dev, at.device) != cudaSuccess) {
            cudaGetLastError();
            can = 0;
        }
        if (!can)
            return fail(CP_ERR_ARG, "%s lives on device %d, which device %d cannot address", name,
                        at.device, dev);
    }
    return CP_OK;
}

cp_status check_align(const void* p, int bytes, const char* name)
{
    if (((uintptr_t)p) % (uintptr_t)bytes != 0)
        return fail(CP_ERR_ALIGN, "%s is not %d-byte aligned", name, bytes);
    return CP_OK;
}

struct Span {
    uintptr_t lo, hi;   // [lo, hi)
    const char* name;
};

bool overlaps(const Span& a, const Span& b) { return a.lo < b.hi && b.lo < a.hi; }

// Byte span of a strided [W][T][H] (x inner elements) view.
Span strided_span(const void* base, int64_t W, int64_t T, int64_t H, int64_t inner,
                  cp_strides3 st, int64_t esize, const char* name)
{
    const int64_t last = (W - 1) * st.r + (T - 1) * st.t + (H - 1) * st.h + inner;
    return {(uintptr_t)base, (uintptr_t)base + (uintptr_t)(last * esize), name};
}

Span dense_span(const void* base, int64_t bytes, const char* name)
{
    return {(uintptr_t)base, (uintptr_t)base + (uintptr_t)bytes, name};
}

cp_status check_no_alias(const Span* in, int nin, const Span* out, int nout)
{
    for (int i = 0; i < nout; ++i) {
        for (int k = 0; k < nin; ++k)
            if (overlaps(out[i], in[k]))
                return fail(CP_ERR_ALIAS, "output %s overlaps input %s", out[i].name, in[k].name);
        for (int k = i + 1; k < nout; ++k)
            if (overlaps(out[i], out[k]))
                return fail(CP_ERR_ALIAS, "outputs %s and %s overlap", out[i].name, out[k].name);
    }
    return CP_OK;
}

cp_status check_strides(cp_strides3 st, bool payload, const char* name)
{
    if (st.r < 0 || st.t < 0 || st.h < 0)
        return fail(CP_ERR_ARG, "%s strides must be >= 0", name);
    if (payload && ((st.r | st.t | st.h) & 7))
        return fail(CP_ERR_ALIGN, "%s strides must be multiples of 8 elements (16 bytes)", name);
    return CP_OK;
}

// W, H, D, dtype and total size shared by pack / fused.
cp_status check_dims(int W, int64_t T, int H, int D, cp_dtype dt)
{
    if (W < 1) return fail(CP_ERR_ARG, "W must be >= 1 (got %d)", W);
    if (W > CPLSE_MAX_W) return fail(CP_ERR_UNSUPPORTED, "W = %d exceeds %d", W, CPLSE_MAX_W);
    if (T < 0) return fail(CP_ERR_ARG, "T must be >= 0");
    if (H < 1 || H % W != 0) return fail(CP_ERR_SHAPE, "H = %d must be a positive multiple of W = %d", H, W);
    if (D < 8 || D % 8 != 0) return fail(CP_ERR_SHAPE, "D = %d must be a positive multiple of 8", D);
    if (D > CPLSE_MAX_D) return fail(CP_ERR_UNSUPPORTED, "D = %d exceeds %d", D, CPLSE_MAX_D);
    if (dt != CP_BF16 && dt != CP_FP16) return fail(CP_ERR_ARG, "unknown dtype %d", (int)dt);
    if (T > ((int64_t)1 << 62) / ((int64_t)W * H * D))
        return fail(CP_ERR_SHAPE, "problem size overflows int64");
    return CP_OK;
}

#define TRY(expr)                          \
    do {                                   \
        cp_status st_ = (expr);            \
        if (st_ != CP_OK) return st_;      \
    } while (0)

cp_status launched(cudaError_t e, const char* what)
{
    if (e != cudaSuccess) return fail(CP_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
    return ok();
}

cp_status check_null(const void* p, const char* name)
{
    if (p == nullptr) return fail(CP_ERR_ARG, "%s is NULL", name);
    return CP_OK;
}

// Host-only checks of the two entry points that read (o, smax, ssum).
cp_status check_sources(const void* o, cp_strides3 so, const float* smax, cp_strides3 sm,
                        const float* ssum, cp_strides3 ss)
{
    TRY(check_null(o, "o"));
    TRY(check_null(smax, "smax"));
    TRY(check_null(ssum, "ssum"));
    TRY(check_align(o, 16, "o"));
    TRY(check_align(smax, 4, "smax"));
    TRY(check_align(ssum, 4, "ssum"));
    TRY(check_strides(so, true, "o"));
    TRY(check_strides(sm, false, "smax"));
    TRY(check_strides(ss, false, "ssum"));
    return CP_OK;
}

// Last: every pointer is device memory of the current device (one driver
// query per pointer; everything before this needs no GPU).
cp_status check_devices(const void* const* p, const char* const* names, int n)
{
    for (int i = 0; i < n; ++i) TRY(check_device_ptr(p[i], names[i]));
    return CP_OK;
}

}  // namespace

// The message cp_last_error() returns, for the entry points in other files.
cp_status cplse_set_error(cp_status st, const char* msg)
{
    snprintf(g_err, sizeof g_err, "%s", msg);
    return st;
}

extern "C" {

int cp_abi_version(void) { return CPLSE_ABI_VERSION; }

const char* cp_last_error(void) { return g_err; }

cp_status cp_pack_lse(const void* o, cp_strides3 so, const float* smax, cp_strides3 sm,
                      const float* ssum, cp_strides3 ss, int W, int64_t T, int H, int D,
                      cp_dtype dt, int scatter_dim, void* pkt_o, float* pkt_lse, void* stream)
{
    TRY(check_dims(W, T, H, D, dt));
    if (scatter_dim != 0 && scatter_dim != 1)
        return fail(CP_ERR_ARG, "scatter_dim must be 0 (tokens) or 1 (heads), got %d", scatter_dim);
    if (scatter_dim == 0 && T % W != 0)
        return fail(CP_ERR_SHAPE, "token scatter needs T %% W == 0 (T = %lld, W = %d)", (long long)T, W);
    if (T == 0) return ok();
    TRY(check_sources(o, so, smax, sm, ssum, ss));
    TRY(check_null(pkt_o, "pkt_o"));
    TRY(check_null(pkt_lse, "pkt_lse"));
    TRY(check_align(pkt_o, 16, "pkt_o"));
    TRY(check_align(pkt_lse, 4, "pkt_lse"));
    const int64_t rows = (int64_t)W * T * H;
    const Span in[3] = {strided_span(o, W, T, H, D, so, 2, "o"),
                        strided_span(smax, W, T, H, 1, sm, 4, "smax"),
                        strided_span(ssum, W, T, H, 1, ss, 4, "ssum")};
    const Span out[2] = {dense_span(pkt_o, rows * D * 2, "pkt_o"),
                         dense_span(pkt_lse, rows * 4, "pkt_lse")};
    TRY(check_no_alias(in, 3, out, 2));
    {
        const void* p[5] = {o, smax, ssum, pkt_o, pkt_lse};
        const char* n[5] = {"o", "smax", "ssum", "pkt_o", "pkt_lse"};
        TRY(check_devices(p, n, 5));
    }

    cplse::PackArgs a{};
    a.o = static_cast<const uint16_t*>(o);
    a.so_r = so.r; a.so_t = so.t; a.so_h = so.h;
    a.smax = smax; a.ssum = ssum;
    a.sm_r = sm.r; a.sm_t = sm.t; a.sm_h = sm.h;
    a.ss_r = ss.r; a.ss_t = ss.t; a.ss_h = ss.h;
    a.pkt_o = static_cast<uint16_t*>(pkt_o);
    a.pkt_lse = pkt_lse;
    a.W = W; a.H = H; a.Hc = H / W; a.D = D; a.scatter_dim = scatter_dim;
    a.T = T; a.Tc = T / W;
    a.rows = rows;
    a.nsrc = W;
    return launched(cplse::launch_pack(a, static_cast<cudaStream_t>(stream)), "cp_pack_lse");
}

cp_status cp_lse_materialize(const float* smax, cp_strides3 sm, const float* ssum,
                             cp_strides3 ss, int W, int64_t T, int H, float* lse, void* stream)
{
    TRY(check_dims(W, T, H, 8, CP_BF16));
    if (T == 0) return ok();
    TRY(check_null(smax, "smax"));
    TRY(check_null(ssum, "ssum"));
    TRY(check_null(lse, "lse"));
    TRY(check_align(smax, 4, "smax"));
    TRY(check_align(ssum, 4, "ssum"));
    TRY(check_align(lse, 4, "lse"));
    TRY(check_strides(sm, false, "smax"));
    TRY(check_strides(ss, false, "ssum"));
    const int64_t rows = (int64_t)W * T * H;
    const Span in[2] = {strided_span(smax, W, T, H, 1, sm, 4, "smax"),
                        strided_span(ssum, W, T, H, 1, ss, 4, "ssum")};
    const Span out[1] = {dense_span(lse, rows * 4, "lse")};
    TRY(check_no_alias(in, 2, out, 1));
    {
        const void* p[3] = {smax, ssum, lse};
        const char* n[3] = {"smax", "ssum", "lse"};
        TRY(check_devices(p, n, 3));
    }
    cplse::PackArgs a{};
    a.smax = smax; a.ssum = ssum;
    a.sm_r = sm.r; a.sm_t = sm.t; a.sm_h = sm.h;
    a.ss_r = ss.r; a.ss_t = ss.t; a.ss_h = ss.h;
    a.W = W; a.H = H; a.T = T; a.rows = rows;
    return launched(cplse::launch_lse_materialize(a, lse, static_cast<cudaStream_t>(stream)),
                    "cp_lse_materialize");
}

cp_status cp_pack_from_lse(const void* o, cp_strides3 so, const float* lse, cp_strides3 sl,
                           int W, int64_t T, int H, int D, cp_dtype dt, int scatter_dim,
                           void* pkt_o, float* pkt_lse, void* stream)
{
    TRY(check_dims(W, T, H, D, dt));
    if (scatter_dim != 0 && scatter_dim != 1)
        return fail(CP_ERR_ARG, "scatter_dim must be 0 (tokens) or 1 (heads), got %d", scatter_dim);
    if (scatter_dim == 0 && T % W != 0)
        return fail(CP_ERR_SHAPE, "token scatter needs T %% W == 0 (T = %lld, W = %d)", (long long)T, W);
    if (T == 0) return ok();
    TRY(check_null(o, "o"));
    TRY(check_null(lse, "lse"));
    TRY(check_null(pkt_o, "pkt_o"));
    TRY(check_null(pkt_lse, "pkt_lse"));
    TRY(check_align(o, 16, "o"));
    TRY(check_align(lse, 4, "lse"));
    TRY(check_align(pkt_o, 16, "pkt_o"));
    TRY(check_align(pkt_lse, 4, "pkt_lse"));
    TRY(check_strides(so, true, "o"));
    TRY(check_strides(sl, false, "lse"));
    const int64_t rows = (int64_t)W * T * H;
    const Span in[2] = {strided_span(o, W, T, H, D, so, 2, "o"),
                        strided_span(lse, W, T, H, 1, sl, 4, "lse")};
    const Span out[2] = {dense_span(pkt_o, rows * D * 2, "pkt_o"),
                         dense_span(pkt_lse, rows * 4, "pkt_lse")};
    TRY(check_no_alias(in, 2, out, 2));
    {
        const void* p[4] = {o, lse, pkt_o, pkt_lse};
        const char* n[4] = {"o", "lse", "pkt_o", "pkt_lse"};
        TRY(check_devices(p, n, 4));
    }
    cplse::PackArgs a{};
    a.o = static_cast<const uint16_t*>(o);
    a.so_r = so.r; a.so_t = so.t; a.so_h = so.h;
    a.lse = lse;
    a.sm_r = sl.r; a.sm_t = sl.t; a.sm_h = sl.h;
    a.pkt_o = static_cast<uint16_t*>(pkt_o);
    a.pkt_lse = pkt_lse;
    a.W = W; a.H = H; a.Hc = H / W; a.D = D; a.scatter_dim = scatter_dim;
    a.T = T; a.Tc = T / W;
    a.rows = rows;
    a.nsrc = W;
    return launched(cplse::launch_pack(a, static_cast<cudaStream_t>(stream)), "cp_pack_from_lse");
}

cp_status cp_a2a_local_permute(const void* send, void* recv, int W, int64_t block_bytes,
                               void* stream)
{
    if (W < 1) return fail(CP_ERR_ARG, "W must be >= 1 (got %d)", W);
    if (W > CPLSE_MAX_W) return fail(CP_ERR_UNSUPPORTED, "W = %d exceeds %d", W, CPLSE_MAX_W);
    if (block_bytes < 0) return fail(CP_ERR_ARG, "block_bytes must be >= 0");
    if (block_bytes > ((int64_t)1 << 62) / ((int64_t)W * W))
        return fail(CP_ERR_SHAPE, "problem size overflows int64");
    if (block_bytes == 0) return ok();
    TRY(check_null(send, "send"));
    TRY(check_null(recv, "recv"));
    const int64_t bytes = (int64_t)W * W * block_bytes;
    const Span in[1] = {dense_span(send, bytes, "send")};
    const Span out[1] = {dense_span(recv, bytes, "recv")};
    TRY(check_no_alias(in, 1, out, 1));
    {
        const void* p[2] = {send, recv};
        const char* n[2] = {"send", "recv"};
        TRY(check_devices(p, n, 2));
    }
    return launched(cplse::launch_permute(send, recv, W, block_bytes,
                                          static_cast<cudaStream_t>(stream)),
                    "cp_a2a_local_permute");
}

cp_status cp_lse_combine(const void* recv_o, const float* recv_lse, int W, int64_t T, int Hc,
                         int D, cp_dtype dt, void* out, float* out_lse, void* stream)
{
    if (Hc < 1) return fail(CP_ERR_SHAPE, "Hc must be >= 1 (got %d)", Hc);
    TRY(check_dims(W, T, Hc * W, D, dt));
    if (T == 0) return ok();
    TRY(check_null(recv_o, "recv_o"));
    TRY(check_null(recv_lse, "recv_lse"));
    TRY(check_null(out, "out"));
    TRY(check_null(out_lse, "out_lse"));
    TRY(check_align(recv_o, 16, "recv_o"));
    TRY(check_align(recv_lse, 4, "recv_lse"));
    TRY(check_align(out, 16, "out"));
    TRY(check_align(out_lse, 4, "out_lse"));
    const int64_t N = T * Hc;
    const Span in[2] = {dense_span(recv_o, (int64_t)W * W * N * D * 2, "recv_o"),
                        dense_span(recv_lse, (int64_t)W * W * N * 4, "recv_lse")};
    const Span outs[2] = {dense_span(out, (int64_t)W * N * D * 2, "out"),
                          dense_span(out_lse, (int64_t)W * N * 4, "out_lse")};
    TRY(check_no_alias(in, 2, outs, 2));
    {
        const void* p[4] = {recv_o, recv_lse, out, out_lse};
        const char* n[4] = {"recv_o", "recv_lse", "out", "out_lse"};
        TRY(check_devices(p, n, 4));
    }

    cplse::CombineArgs a{};
    a.src = static_cast<const uint16_t*>(recv_o);
    a.rank_stride = N * D;
    a.lse = recv_lse;
    a.out = static_cast<uint16_t*>(out);
    a.out_lse = out_lse;
    a.W = W; a.H = Hc * W; a.Hc = Hc; a.D = D;
    a.T = T; a.N = N; a.rows = (int64_t)W * N;
    a.dense_rows = 1;
    return launched(cplse::launch_combine_async(a, static_cast<cplse::Dtype>(dt),
                                                static_cast<cudaStream_t>(stream)),
                    "cp_lse_combine");
}

cp_status cp_pack_permute_combine_fused(const void* o, cp_strides3 so, const float* smax,
                                        cp_strides3 sm, const float* ssum, cp_strides3 ss, int W,
                                        int64_t T, int H, int D, cp_dtype dt, int scatter_dim,
                                        void* out, float* out_lse, void* stream)
{
    TRY(check_dims(W, T, H, D, dt));
    if (scatter_dim != 0 && scatter_dim != 1)
        return fail(CP_ERR_ARG, "scatter_dim must be 0 (tokens) or 1 (heads), got %d", scatter_dim);
    if (scatter_dim == 0 && T % W != 0)
        return fail(CP_ERR_SHAPE, "token scatter needs T %% W == 0 (T = %lld, W = %d)", (long long)T, W);
    if (T == 0) return ok();
    TRY(check_sources(o, so, smax, sm, ssum, ss));
    TRY(check_null(out, "out"));
    TRY(check_null(out_lse, "out_lse"));
    TRY(check_align(out, 16, "out"));
    TRY(check_align(out_lse, 4, "out_lse"));
    const int64_t rows = T * H;
    const Span in[3] = {strided_span(o, W, T, H, D, so, 2, "o"),
                        strided_span(smax, W, T, H, 1, sm, 4, "smax"),
                        strided_span(ssum, W, T, H, 1, ss, 4, "ssum")};
    const Span outs[2] = {dense_span(out, rows * D * 2, "out"),
                          dense_span(out_lse, rows * 4, "out_lse")};
    TRY(check_no_alias(in, 3, outs, 2));
    {
        const void* p[5] = {o, smax, ssum, out, out_lse};
        const char* n[5] = {"o", "smax", "ssum", "out", "out_lse"};
        TRY(check_devices(p, n, 5));
    }

    cplse::CombineArgs a{};
    a.src = static_cast<const uint16_t*>(o);
    a.rank_stride = so.r;
    a.so_t = so.t; a.so_h = so.h;
    a.smax = smax; a.ssum = ssum;
    a.sm_r = sm.r; a.sm_t = sm.t; a.sm_h = sm.h;
    a.ss_r = ss.r; a.ss_t = ss.t; a.ss_h = ss.h;
    a.out = static_cast<uint16_t*>(out);
    a.out_lse = out_lse;
    a.W = W; a.H = H; a.Hc = H / W; a.D = D;
    a.T = T; a.N = T * (H / W); a.rows = rows;
    a.dense_rows = (so.h == D && so.t == (int64_t)H * D) ? 1 : 0;
    a.token_scatter = scatter_dim == 0 ? 1 : 0;
    return launched(cplse::launch_fused_async(a, static_cast<cplse::Dtype>(dt),
                                              static_cast<cudaStream_t>(stream)),
                    "cp_pack_permute_combine_fused");
}

cp_status cp_pack_lse_rank(const void* o, cp_strides3 so, const float* smax, cp_strides3 sm,
                           const float* ssum, cp_strides3 ss, int W, int64_t T, int H, int D,
                           cp_dtype dt, int scatter_dim, void* pkt_o, float* pkt_lse, void* stream)
{
    TRY(check_dims(W, T, H, D, dt));
    if (scatter_dim != 0 && scatter_dim != 1)
        return fail(CP_ERR_ARG, "scatter_dim must be 0 (tokens) or 1 (heads), got %d", scatter_dim);
    if (scatter_dim == 0 && T % W != 0)
        return fail(CP_ERR_SHAPE, "token scatter needs T %% W == 0 (T = %lld, W = %d)", (long long)T, W);
    if (T == 0) return ok();
    so.r = sm.r = ss.r = 0;                    // one source plane
    TRY(check_sources(o, so, smax, sm, ssum, ss));
    TRY(check_null(pkt_o, "pkt_o"));
    TRY(check_null(pkt_lse, "pkt_lse"));
    TRY(check_align(pkt_o, 16, "pkt_o"));
    TRY(check_align(pkt_lse, 4, "pkt_lse"));
    const int64_t rows = T * H;
    const Span in[3] = {strided_span(o, 1, T, H, D, so, 2, "o"),
                        strided_span(smax, 1, T, H, 1, sm, 4, "smax"),
                        strided_span(ssum, 1, T, H, 1, ss, 4, "ssum")};
    const Span out[2] = {dense_span(pkt_o, rows * D * 2, "pkt_o"),
                         dense_span(pkt_lse, rows * 4, "pkt_lse")};
    TRY(check_no_alias(in, 3, out, 2));
    {
        const void* p[5] = {o, smax, ssum, pkt_o, pkt_lse};
        const char* n[5] = {"o", "smax", "ssum", "pkt_o", "pkt_lse"};
        TRY(check_devices(p, n, 5));
    }
    cplse::PackArgs a{};
    a.o = static_cast<const uint16_t*>(o);
    a.so_r = 0; a.so_t = so.t; a.so_h = so.h;
    a.smax = smax; a.ssum = ssum;
    a.sm_r = 0; a.sm_t = sm.t; a.sm_h = sm.h;
    a.ss_r = 0; a.ss_t = ss.t; a.ss_h = ss.h;
    a.pkt_o = static_cast<uint16_t*>(pkt_o);
    a.pkt_lse = pkt_lse;
    a.W = W; a.H = H; a.Hc = H / W; a.D = D; a.scatter_dim = scatter_dim;
    a.T = T; a.Tc = T / W;
    a.rows = rows;
    a.nsrc = 1;
    return launched(cplse::launch_pack(a, static_cast<cudaStream_t>(stream)), "cp_pack_lse_rank");
}

cp_status cp_lse_combine_rank(const void* recv_o, const float* recv_lse, int W, int64_t T, int Hc,
                              int D, cp_dtype dt, void* out, float* out_lse, void* stream)
{
    if (Hc < 1) return fail(CP_ERR_SHAPE, "Hc must be >= 1 (got %d)", Hc);
    TRY(check_dims(W, T, Hc * W, D, dt));
    if (T == 0) return ok();
    TRY(check_null(recv_o, "recv_o"));
    TRY(check_null(recv_lse, "recv_lse"));
    TRY(check_null(out, "out"));
    TRY(check_null(out_lse, "out_lse"));
    TRY(check_align(recv_o, 16, "recv_o"));
    TRY(check_align(recv_lse, 4, "recv_lse"));
    TRY(check_align(out, 16, "out"));
    TRY(check_align(out_lse, 4, "out_lse"));
    const int64_t N = T * Hc;
    const Span in[2] = {dense_span(recv_o, (int64_t)W * N * D * 2, "recv_o"),
                        dense_span(recv_lse, (int64_t)W * N * 4, "recv_lse")};
    const Span outs[2] = {dense_span(out, N * D * 2, "out"), dense_span(out_lse, N * 4, "out_lse")};
    TRY(check_no_alias(in, 2, outs, 2));
    {
        const void* p[4] = {recv_o, recv_lse, out, out_lse};
        const char* n[4] = {"recv_o", "recv_lse", "out", "out_lse"};
        TRY(check_devices(p, n, 4));
    }
    // the received packet of one destination is destination 0 of a W-rank packet
    cplse::CombineArgs a{};
    a.src = static_cast<const uint16_t*>(recv_o);
    a.rank_stride = N * D;
    a.lse = recv_lse;
    a.out = static_cast<uint16_t*>(out);
    a.out_lse = out_lse;
    a.W = W; a.H = Hc * W; a.Hc = Hc; a.D = D;
    a.T = T; a.N = N; a.rows = N;
    a.dense_rows = 1;
    return launched(cplse::launch_combine_async(a, static_cast<cplse::Dtype>(dt),
                                                static_cast<cudaStream_t>(stream)),
                    "cp_lse_combine_rank");
}

cp_status cp_pull_combine(const void* const* o, cp_strides3 so, const float* const* smax,
                          cp_strides3 sm, const float* const* ssum, cp_strides3 ss, int W,
                          int64_t T, int H, int D, cp_dtype dt, int scatter_dim, int dst,
                          void* out, float* out_lse, void* stream)
{
    TRY(check_dims(W, T, H, D, dt));
    if (scatter_dim != 0 && scatter_dim != 1)
        return fail(CP_ERR_ARG, "scatter_dim must be 0 (tokens) or 1 (heads), got %d", scatter_dim);
    if (scatter_dim == 0 && T % W != 0)
        return fail(CP_ERR_SHAPE, "token scatter needs T %% W == 0 (T = %lld, W = %d)", (long long)T, W);
    if (dst < 0 || dst >= W) return fail(CP_ERR_ARG, "dst = %d is not a rank of 0..%d", dst, W - 1);
    if (T == 0) return ok();
    TRY(check_null(o, "o"));
    TRY(check_null(smax, "smax"));
    TRY(check_null(ssum, "ssum"));
    so.r = sm.r = ss.r = 0;                    // every rank's plane has its own base
    char nm[3][16];
    for (int r = 0; r < W; ++r) {
        snprintf(nm[0], sizeof nm[0], "o[%d]", r);
        snprintf(nm[1], sizeof nm[1], "smax[%d]", r);
        snprintf(nm[2], sizeof nm[2], "ssum[%d]", r);
        TRY(check_null(o[r], nm[0]));
        TRY(check_null(smax[r], nm[1]));
        TRY(check_null(ssum[r], nm[2]));
        TRY(check_align(o[r], 16, nm[0]));
        TRY(check_align(smax[r], 4, nm[1]));
        TRY(check_align(ssum[r], 4, nm[2]));
    }
    TRY(check_strides(so, true, "o"));
    TRY(check_strides(sm, false, "smax"));
    TRY(check_strides(ss, false, "ssum"));
    TRY(check_null(out, "out"));
    TRY(check_null(out_lse, "out_lse"));
    TRY(check_align(out, 16, "out"));
    TRY(check_align(out_lse, 4, "out_lse"));
    const int Hc = H / W;
    const int64_t Tc = T / W;
    const int64_t rows = scatter_dim == 1 ? T * Hc : Tc * H;
    const Span outs[2] = {dense_span(out, rows * D * 2, "out"),
                          dense_span(out_lse, rows * 4, "out_lse")};
    for (int r = 0; r < W; ++r) {
        const Span in[3] = {strided_span(o[r], 1, T, H, D, so, 2, "o[r]"),
                            strided_span(smax[r], 1, T, H, 1, sm, 4, "smax[r]"),
                            strided_span(ssum[r], 1, T, H, 1, ss, 4, "ssum[r]")};
        TRY(check_no_alias(in, 3, outs, 2));
    }
    {
        const void* p[2] = {out, out_lse};
        const char* n[2] = {"out", "out_lse"};
        TRY(check_devices(p, n, 2));
    }
    for (int r = 0; r < W; ++r) {
        snprintf(nm[0], sizeof nm[0], "o[%d]", r);
        snprintf(nm[1], sizeof nm[1], "smax[%d]", r);
        snprintf(nm[2], sizeof nm[2], "ssum[%d]", r);
        TRY(check_addressable_ptr(o[r], nm[0]));
        TRY(check_addressable_ptr(smax[r], nm[1]));
        TRY(check_addressable_ptr(ssum[r], nm[2]));
    }
    cplse::PullArgs a{};
    for (int r = 0; r < W; ++r) {
        a.o[r] = static_cast<const uint16_t*>(o[r]);
        a.smax[r] = smax[r];
        a.ssum[r] = ssum[r];
    }
    a.so_t = so.t; a.so_h = so.h;
    a.sm_t = sm.t; a.sm_h = sm.h;
    a.ss_t = ss.t; a.ss_h = ss.h;
    a.out = static_cast<uint16_t*>(out);
    a.out_lse = out_lse;
    a.W = W; a.H = H; a.Hc = Hc; a.D = D;
    a.dst = dst;
    a.token_scatter = scatter_dim == 0 ? 1 : 0;
    a.T = T; a.Tc = Tc;
    a.rows = rows;
    return launched(cplse::launch_pull_combine(a, static_cast<cplse::Dtype>(dt),
                                               static_cast<cudaStream_t>(stream)),
                    "cp_pull_combine");
}

static cp_status ulysses(const void* in, void* out, int W, int B, int64_t S_local, int H, int D,
                         int elem_bytes, void* stream, int mode, const char* what)
{
    if (W < 1) return fail(CP_ERR_ARG, "W must be >= 1 (got %d)", W);
    if (W > CPLSE_MAX_W) return fail(CP_ERR_UNSUPPORTED, "W = %d exceeds %d", W, CPLSE_MAX_W);
    if (B < 0 || S_local < 0) return fail(CP_ERR_ARG, "B and S_local must be >= 0");
    if (H < 1 || H % W != 0) return fail(CP_ERR_SHAPE, "H = %d must be a positive multiple of W = %d", H, W);
    if (D < 1) return fail(CP_ERR_SHAPE, "D must be >= 1");
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
        return fail(CP_ERR_ARG, "elem_bytes must be 1, 2, 4 or 8 (got %d)", elem_bytes);
    const int64_t per_rank = (int64_t)B * H * D * elem_bytes;
    if (S_local > 0 && per_rank > 0 && S_local > ((int64_t)1 << 62) / ((int64_t)W * W * per_rank))
        return fail(CP_ERR_SHAPE, "problem size overflows int64");
    if (B == 0 || S_local == 0) return ok();
    TRY(check_null(in, "in"));
    TRY(check_null(out, "out"));
    const int64_t bytes = (int64_t)W * S_local * per_rank;   // W ranks x [B][S_l][H][D]
    const Span ins[1] = {dense_span(in, bytes, "in")};
    const Span outs[1] = {dense_span(out, bytes, "out")};
    TRY(check_no_alias(ins, 1, outs, 1));
    {
        const void* p[2] = {in, out};
        const char* n[2] = {"in", "out"};
        TRY(check_devices(p, n, 2));
    }
    cplse::UlyssesArgs a{};
    a.in = in; a.out = out;
    a.W = W; a.B = B; a.H = H; a.Hc = H / W;
    a.S_l = S_local; a.S = S_local * W;
    a.chunk_bytes = (int64_t)(H / W) * D * elem_bytes;
    a.nchunks = (int64_t)W * B * S_local * W;
    a.mode = mode;
    return launched(cplse::launch_ulysses(a, static_cast<cudaStream_t>(stream)), what);
}

static cp_status ulysses_pull(const void* const* in, void* out, int W, int B, int64_t S_local,
                              int H, int D, int elem_bytes, int dst, void* stream, int mode,
                              const char* what)
{
    if (W < 1) return fail(CP_ERR_ARG, "W must be >= 1 (got %d)", W);
    if (W > CPLSE_MAX_W) return fail(CP_ERR_UNSUPPORTED, "W = %d exceeds %d", W, CPLSE_MAX_W);
    if (B < 0 || S_local < 0) return fail(CP_ERR_ARG, "B and S_local must be >= 0");
    if (B > 65535) return fail(CP_ERR_UNSUPPORTED, "B = %d exceeds 65535", B);
    if (H < 1 || H % W != 0) return fail(CP_ERR_SHAPE, "H = %d must be a positive multiple of W = %d", H, W);
    if (D < 1) return fail(CP_ERR_SHAPE, "D must be >= 1");
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
        return fail(CP_ERR_ARG, "elem_bytes must be 1, 2, 4 or 8 (got %d)", elem_bytes);
    if (dst < 0 || dst >= W) return fail(CP_ERR_ARG, "dst = %d is not a rank of 0..%d", dst, W - 1);
    const int64_t per_rank = (int64_t)B * H * D * elem_bytes;
    if (S_local > 0 && per_rank > 0 && S_local > ((int64_t)1 << 62) / ((int64_t)W * per_rank))
        return fail(CP_ERR_SHAPE, "problem size overflows int64");
    if (B == 0 || S_local == 0) return ok();
    TRY(check_null(in, "in"));
    TRY(check_null(out, "out"));
    const int64_t bytes = S_local * per_rank;      // one rank's tensor (either layout)
    const Span outs[1] = {dense_span(out, bytes, "out")};
    char nm[16];
    for (int r = 0; r < W; ++r) {
        snprintf(nm, sizeof nm, "in[%d]", r);
        TRY(check_null(in[r], nm));
        const Span ins[1] = {dense_span(in[r], bytes, "in[r]")};
        TRY(check_no_alias(ins, 1, outs, 1));
    }
    {
        const void* p[1] = {out};
        const char* n[1] = {"out"};
        TRY(check_devices(p, n, 1));
    }
    for (int r = 0; r < W; ++r) {
        snprintf(nm, sizeof nm, "in[%d]", r);
        TRY(check_addressable_ptr(in[r], nm));
    }
    cplse::UlyssesArgs a{};
    a.in = nullptr; a.out = out;
    a.W = W; a.B = B; a.H = H; a.Hc = H / W;
    a.S_l = S_local; a.S = S_local * W;
    a.chunk_bytes = (int64_t)(H / W) * D * elem_bytes;
    a.nchunks = (int64_t)W * B * S_local;
    a.mode = mode;
    a.pull = 1;
    a.dst = dst;
    for (int r = 0; r < W; ++r) a.ins[r] = in[r];
    return launched(cplse::launch_ulysses(a, static_cast<cudaStream_t>(stream)), what);
}

cp_status ulysses_seq2head_pull(const void* const* in, void* out, int W, int B, int64_t S_local,
                                int H, int D, int elem_bytes, int dst, void* stream)
{
    return ulysses_pull(in, out, W, B, S_local, H, D, elem_bytes, dst, stream, 0,
                        "ulysses_seq2head_pull");
}

cp_status ulysses_head2seq_pull(const void* const* in, void* out, int W, int B, int64_t S_local,
                                int H, int D, int elem_bytes, int dst, void* stream)
{
    return ulysses_pull(in, out, W, B, S_local, H, D, elem_bytes, dst, stream, 1,
                        "ulysses_head2seq_pull");
}

cp_status ulysses_seq2head(const void* in, void* out, int W, int B, int64_t S_local, int H, int D,
                           int elem_bytes, void* stream)
{
    return ulysses(in, out, W, B, S_local, H, D, elem_bytes, stream, 0, "ulysses_seq2head");
}

cp_status ulysses_head2seq(const void* in, void* out, int W, int B, int64_t S_local, int H, int D,
                           int elem_bytes, void* stream)
{
    return ulysses(in, out, W, B, S_local, H, D, elem_bytes, stream, 1, "ulysses_head2seq");
}

}  // extern "C"
