// api.cu -- the extern "C" entry points of libhyena_b200.so: argument
// validation, path selection and launch.  See include/hyena.h for semantics.
#include <cstdint>
#include <cstring>

#include "chunk_lanes.h"
#include "kernels.h"
#include "host_pipeline.h"
#include "resident.cuh"
#include "status.h"
#include "twiddle.h"

using namespace hy;

namespace {

constexpr int kMaxResidentLogM = 14;   // M = 16384 complex points on chip

bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }
int ilog2(int64_t x) {
    int r = 0;
    while ((int64_t(1) << r) < x) ++r;
    return r;
}
int64_t spectrum_m(int64_t L) {
    int64_t m = 16;
    while (m < L) m *= 2;
    return m;
}
bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }
size_t dt_size(hy_dtype dt) { return dt == HY_BF16 ? 2 : 4; }
bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b) return false;
    const char *pa = (const char *)a, *pb = (const char *)b;
    return pa < pb + nb && pb < pa + na;
}

hy_status prologue(cudaStream_t) {
    clear_error();
    hy_status st = tw_ensure_device();
    // the chunk pipelines' second stream is made here, with the first call
    // on the device (before any capture), not inside a captured call
    if (st == HY_OK) chunk_lanes_of_device();
    return st;
}

// Shared body of hyena_fftconv / hyena_operator (1-D, causal).
hy_status run_chain(int K, int B, int D, int L, hy_dtype dt, const void *v, const void *const *gates,
                    const hy_c32 *const *H, const float *const *Dskip, void *y, void *ws,
                    size_t ws_bytes, cudaStream_t stream, const char *who) {
    if (B < 1 || D < 1 || L < 1) return set_error(HY_ERR_INVALID_ARG, "%s: B, D, L must be >= 1", who);
    if (dt != HY_F32 && dt != HY_BF16) return set_error(HY_ERR_INVALID_ARG, "%s: unknown dtype", who);
    if (!v || !y) return set_error(HY_ERR_INVALID_ARG, "%s: null signal pointer", who);
    const size_t esz = dt_size(dt);
    const size_t nbytes = (size_t)B * D * L * esz;
    const size_t al = (L % 2 == 0) ? 2 * esz : esz;
    if (!aligned(v, al) || !aligned(y, al))
        return set_error(HY_ERR_INVALID_ARG, "%s: signals must be %zu-byte aligned", who, al);
    if (overlap(v, nbytes, y, nbytes)) return set_error(HY_ERR_INVALID_ARG, "%s: y aliases the input", who);
    const int64_t M = spectrum_m(L);
    for (int k = 0; k < K; ++k) {
        if (!H[k]) return set_error(HY_ERR_INVALID_ARG, "%s: spectrum %d is null", who, k);
        if (!aligned(H[k], 8)) return set_error(HY_ERR_INVALID_ARG, "%s: spectrum %d misaligned", who, k);
        if (gates[k]) {
            if (!aligned(gates[k], al)) return set_error(HY_ERR_INVALID_ARG, "%s: gate %d misaligned", who, k);
            if (overlap(gates[k], nbytes, y, nbytes))
                return set_error(HY_ERR_INVALID_ARG, "%s: y aliases gate %d", who, k);
        }
        if (Dskip && Dskip[k] && overlap(Dskip[k], (size_t)D * 4, y, nbytes))
            return set_error(HY_ERR_INVALID_ARG, "%s: y aliases Dskip %d", who, k);
    }
    const int log_m = ilog2(M);
    if (log_m <= kMaxResidentLogM) {
        hy_status st = prologue(stream);
        if (st != HY_OK) return st;
        ResidentParams p{};
        p.n_rows = (int64_t)B * D;
        p.L = L;
        p.K = K;
        p.B = B;
        p.D = D;
        p.remap = 1;
        p.u = v;
        for (int k = 0; k < K; ++k) {
            p.gate[k] = gates[k];
            p.spec[k] = reinterpret_cast<const float2 *>(H[k]);
            p.skip[k] = Dskip ? Dskip[k] : nullptr;
        }
        p.spec_row_stride = M + 1;
        p.sdiv = 1;
        p.smod = D;
        p.spec_batch_stride = 0;
        p.y = y;
        p.scale = (float)(1.0 / (4.0 * (double)M));
        return launch_resident_conv(p, log_m, dt, false, stream);
    }
    // long sequences: multi-pass path
    LongConvArgs a{};
    a.K = K;
    a.B = B;
    a.D = D;
    a.L = L;
    a.log_mc = log_m;
    a.dt = dt;
    a.u = v;
    for (int k = 0; k < K; ++k) {
        a.gate[k] = gates[k];
        a.spec[k] = reinterpret_cast<const float2 *>(H[k]);
        a.skip[k] = Dskip ? Dskip[k] : nullptr;
    }
    a.y = y;
    a.ws = ws;
    a.ws_bytes = ws_bytes;
    const size_t need = long_conv_workspace_min(B, D, log_m);
    if (need == 0) return set_error(HY_ERR_UNSUPPORTED, "%s: L=%d is beyond the supported length", who, L);
    if (!ws || ws_bytes < need)
        return set_error(HY_ERR_WORKSPACE, "%s: needs %zu workspace bytes, got %zu", who, need, ws ? ws_bytes : (size_t)0);
    if (!aligned(ws, 256)) return set_error(HY_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
    hy_status st = prologue(stream);
    if (st != HY_OK) return st;
    return launch_long_conv(a, stream);
}

}  // namespace

extern "C" {

int hyena_abi_version(void) { return HYENA_ABI_VERSION; }

const char *hyena_status_string(hy_status s) {
    switch (s) {
        case HY_OK: return "HY_OK";
        case HY_ERR_INVALID_ARG: return "HY_ERR_INVALID_ARG";
        case HY_ERR_UNSUPPORTED: return "HY_ERR_UNSUPPORTED";
        case HY_ERR_WORKSPACE: return "HY_ERR_WORKSPACE";
        case HY_ERR_CUDA: return "HY_ERR_CUDA";
        case HY_ERR_TIMEOUT: return "HY_ERR_TIMEOUT";
    }
    return "unknown status";
}

hy_status hyena_init(void) {
    return prologue(nullptr);
}

int64_t hyena_spectrum_bins(int64_t L) {
    if (L < 1) return 0;
    return spectrum_m(L) + 1;
}

hy_status hyena_filter_gen(const hy_filter_desc *d, float *h, void *stream) {
    clear_error();
    if (!d || !h) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: null desc or output");
    if (d->ndim != 1 && d->ndim != 3) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: ndim must be 1 or 3");
    if (d->n_layers < 1 || d->n_layers > 4) return set_error(HY_ERR_UNSUPPORTED, "hyena_filter_gen: n_layers must be 1..4");
    if (!d->widths || !d->W || !d->b || !d->alpha) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: null parameter array");
    if (d->n_freq < 0 || d->n_sets < 1) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: bad n_freq or n_sets");
    if (d->act != HY_ACT_SILU && d->act != HY_ACT_IDENTITY && d->act != HY_ACT_SINE)
        return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: bad activation");
    if (d->window != HY_WIN_EXP && d->window != HY_WIN_GAUSS) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: bad window");
    if ((d->film_gamma == nullptr) != (d->film_beta == nullptr))
        return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: film_gamma and film_beta go together");
    if (d->film_gamma && d->n_layers < 2) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: FiLM needs a hidden layer");
    if (!d->film_gamma && d->n_sets != 1) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: n_sets > 1 needs FiLM");
    for (int l = 0; l <= d->n_layers; ++l)
        if (d->widths[l] < 1) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: width %d < 1", l);
    for (int l = 0; l < d->n_layers; ++l)
        if (!d->W[l] || !d->b[l]) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: null weight of layer %d", l);
    if (d->ndim == 1) {
        if (d->L < 1) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: L must be >= 1");
        if (d->widths[0] != (d->include_t ? 1 : 0) + 2 * d->n_freq)
            return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: widths[0] must equal include_t + 2F");
        if (d->n_freq < 1 && !d->include_t) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: empty encoding");
    } else {
        if (!is_pow2(d->grid) || d->grid < 2 || d->grid > 64)
            return set_error(HY_ERR_UNSUPPORTED, "hyena_filter_gen: grid must be a power of two in [2, 64]");
        if (d->widths[0] != 6 * d->n_freq || d->n_freq < 1)
            return set_error(HY_ERR_INVALID_ARG, "hyena_filter_gen: widths[0] must equal 6F (F >= 1)");
    }
    hy_status st = tw_ensure_device();
    if (st != HY_OK) return st;
    return launch_filter_gen(*d, h, (cudaStream_t)stream);
}

size_t hyena_filter_spectrum_workspace(int64_t rows, int ndim, const int *dims, int circular) {
    if (rows < 1 || !dims) return 0;
    if (ndim == 1) {
        if (circular) return 0;
        const int log_m = ilog2(spectrum_m(dims[0]));
        return log_m <= kMaxResidentLogM ? 0 : long_spectrum_workspace(rows, log_m);
    }
    if (ndim == 3) {
        int S[3];
        for (int a = 0; a < 3; ++a) S[a] = circular ? dims[a] : 2 * dims[a];
        return nd_spectrum_workspace(rows, S);
    }
    return 0;
}

hy_status hyena_filter_spectrum(int64_t rows, int ndim, const int *dims, int circular, const float *h,
                                hy_c32 *H, void *ws, size_t ws_bytes, void *stream) {
    clear_error();
    if (rows < 1 || !dims || !h || !H) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_spectrum: bad rows or null pointer");
    if (!aligned(h, 8) || !aligned(H, 8)) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_spectrum: pointers must be 8-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    if (ndim == 1) {
        const int64_t L = dims[0];
        if (L < 1) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_spectrum: L must be >= 1");
        const int64_t bins = circular ? L / 2 + 1 : spectrum_m(L) + 1;
        if (overlap(h, (size_t)rows * L * 4, H, (size_t)rows * bins * 8))
            return set_error(HY_ERR_INVALID_ARG, "hyena_filter_spectrum: H aliases h");
        if (circular) {
            if (!is_pow2(L) || L < 32 || L > 32768)
                return set_error(HY_ERR_UNSUPPORTED, "hyena_filter_spectrum: circular L must be a power of two in [32, 32768]");
            hy_status st = prologue(s);
            if (st != HY_OK) return st;
            return launch_spectrum_1d(rows, (int)L, ilog2(L / 2), true, h, reinterpret_cast<float2 *>(H), s);
        }
        const int log_m = ilog2(spectrum_m(L));
        if (log_m <= kMaxResidentLogM) {
            hy_status st = prologue(s);
            if (st != HY_OK) return st;
            return launch_spectrum_1d(rows, (int)L, log_m, false, h, reinterpret_cast<float2 *>(H), s);
        }
        const size_t need = long_spectrum_workspace_min(rows, log_m);
        if (need == 0) return set_error(HY_ERR_UNSUPPORTED, "hyena_filter_spectrum: L=%lld beyond the supported length", (long long)L);
        if (!ws || ws_bytes < need)
            return set_error(HY_ERR_WORKSPACE, "hyena_filter_spectrum: needs %zu workspace bytes", need);
        if (!aligned(ws, 256)) return set_error(HY_ERR_INVALID_ARG, "hyena_filter_spectrum: workspace must be 256-byte aligned");
        hy_status st = prologue(s);
        if (st != HY_OK) return st;
        return launch_long_spectrum(rows, L, log_m, h, reinterpret_cast<float2 *>(H), ws, ws_bytes, s);
    }
    if (ndim == 3) {
        int S[3];
        for (int a = 0; a < 3; ++a) {
            if (!is_pow2(dims[a]) || dims[a] < 4 || dims[a] > 128)
                return set_error(HY_ERR_UNSUPPORTED, "hyena_filter_spectrum: grid edges must be powers of two in [4, 128]");
            S[a] = circular ? dims[a] : 2 * dims[a];
            if (S[a] > 128) return set_error(HY_ERR_UNSUPPORTED, "hyena_filter_spectrum: transform edge %d > 128", S[a]);
        }
        const size_t need = nd_spectrum_workspace(rows, S, true);
        if (need > 0 && (!ws || ws_bytes < need))
            return set_error(HY_ERR_WORKSPACE, "hyena_filter_spectrum: needs %zu workspace bytes", need);
        hy_status st = prologue(s);
        if (st != HY_OK) return st;
        return launch_nd_spectrum(rows, S, h, reinterpret_cast<float2 *>(H), ws, ws_bytes, s);
    }
    return set_error(HY_ERR_INVALID_ARG, "hyena_filter_spectrum: ndim must be 1 or 3");
}

hy_status hyena_fftconv(int B, int D, int L, hy_dtype dt, const void *u, const hy_c32 *H, const float *Dskip,
                        const void *gate, void *y, void *ws, size_t ws_bytes, void *stream) {
    clear_error();
    const void *gates[1] = {gate};
    const hy_c32 *Hs[1] = {H};
    const float *sk[1] = {Dskip};
    return run_chain(1, B, D, L, dt, u, gates, Hs, sk, y, ws, ws_bytes, (cudaStream_t)stream, "hyena_fftconv");
}

size_t hyena_operator_workspace(int order, int B, int D, int L, hy_dtype dt) {
    (void)dt;
    if (order < 2 || order - 1 > kMaxOrders || B < 1 || D < 1 || L < 1) return 0;
    const int log_m = ilog2(spectrum_m(L));
    if (log_m <= kMaxResidentLogM) return 0;
    return long_conv_workspace(B, D, log_m, order - 1);
}

hy_status hyena_operator(int order, int B, int D, int L, hy_dtype dt, const void *v, const void *const *x,
                         const hy_c32 *const *H, const float *const *Dskip, void *y, void *ws, size_t ws_bytes,
                         void *stream) {
    clear_error();
    if (order < 2 || order - 1 > kMaxOrders)
        return set_error(HY_ERR_UNSUPPORTED, "hyena_operator: order must be 2..%d", kMaxOrders + 1);
    if (!x || !H) return set_error(HY_ERR_INVALID_ARG, "hyena_operator: null x or H array");
    for (int k = 0; k < order - 1; ++k)
        if (!x[k]) return set_error(HY_ERR_INVALID_ARG, "hyena_operator: x[%d] is null", k);
    return run_chain(order - 1, B, D, L, dt, v, x, H, Dskip, y, ws, ws_bytes, (cudaStream_t)stream, "hyena_operator");
}

size_t hyena_nd_conv_workspace(int ndim, const int *dims, int B, int D, int circular) {
    if (ndim != 3 || !dims || B < 1 || D < 1) return 0;
    int g[3] = {dims[0], dims[1], dims[2]};
    return nd_conv_workspace(g, circular, B, D);
}

hy_status hyena_nd_conv(int ndim, const int *dims, int B, int D, int circular, const float *u, const hy_c32 *H,
                        int64_t H_batch_stride, const float *Dskip, const float *gate, float *y, void *ws,
                        size_t ws_bytes, void *stream) {
    clear_error();
    if (ndim != 3) return set_error(HY_ERR_UNSUPPORTED, "hyena_nd_conv: only ndim = 3 is built");
    if (!dims || !u || !H || !y) return set_error(HY_ERR_INVALID_ARG, "hyena_nd_conv: null pointer");
    if (B < 1 || D < 1 || H_batch_stride < 0) return set_error(HY_ERR_INVALID_ARG, "hyena_nd_conv: bad B, D or stride");
    NDArgs a{};
    for (int i = 0; i < 3; ++i) {
        if (!is_pow2(dims[i]) || dims[i] < 4 || dims[i] > 128)
            return set_error(HY_ERR_UNSUPPORTED, "hyena_nd_conv: grid edges must be powers of two in [4, 128]");
        a.g[i] = dims[i];
        a.S[i] = circular ? dims[i] : 2 * dims[i];
        if (a.S[i] > 128) return set_error(HY_ERR_UNSUPPORTED, "hyena_nd_conv: transform edge %d > 128", a.S[i]);
    }
    const size_t vox = (size_t)dims[0] * dims[1] * dims[2];
    const size_t nbytes = (size_t)B * D * vox * 4;
    if (!aligned(u, 16) || !aligned(y, 16) || (gate && !aligned(gate, 16)) || !aligned(H, 8))
        return set_error(HY_ERR_INVALID_ARG, "hyena_nd_conv: signals must be 16-byte aligned");
    if (overlap(u, nbytes, y, nbytes) || overlap(gate, nbytes, y, nbytes))
        return set_error(HY_ERR_INVALID_ARG, "hyena_nd_conv: y aliases an input");
    a.circular = circular ? 1 : 0;
    a.B = B;
    a.D = D;
    a.u = u;
    a.H = reinterpret_cast<const float2 *>(H);
    a.H_batch_stride = H_batch_stride;
    a.skip = Dskip;
    a.gate = gate;
    a.y = y;
    a.ws = ws;
    a.ws_bytes = ws_bytes;
    const size_t need = nd_conv_workspace(a.g, a.circular, B, D, true);
    if (need > 0 && (!ws || ws_bytes < need))
        return set_error(HY_ERR_WORKSPACE, "hyena_nd_conv: needs %zu workspace bytes, got %zu", need, ws ? ws_bytes : (size_t)0);
    if (ws && !aligned(ws, 256)) return set_error(HY_ERR_INVALID_ARG, "hyena_nd_conv: workspace must be 256-byte aligned");
    hy_status st = prologue((cudaStream_t)stream);
    if (st != HY_OK) return st;
    return launch_nd_conv(a, (cudaStream_t)stream);
}

hy_status spectral_gate(int B, int H, int Dh, int L, hy_dtype dt, const void *x, const hy_c32 *g,
                        int64_t g_batch_stride, const void *x2, void *y, void *stream) {
    clear_error();
    if (B < 1 || H < 1 || Dh < 1) return set_error(HY_ERR_INVALID_ARG, "spectral_gate: B, H, Dh must be >= 1");
    if (dt != HY_F32 && dt != HY_BF16) return set_error(HY_ERR_INVALID_ARG, "spectral_gate: unknown dtype");
    if (!is_pow2(L) || L < 32 || L > 32768)
        return set_error(HY_ERR_UNSUPPORTED, "spectral_gate: L must be a power of two in [32, 32768]");
    if (!x || !g || !y) return set_error(HY_ERR_INVALID_ARG, "spectral_gate: null pointer");
    if (g_batch_stride < 0) return set_error(HY_ERR_INVALID_ARG, "spectral_gate: negative gate stride");
    const size_t esz = dt_size(dt);
    const size_t nbytes = (size_t)B * H * Dh * L * esz;
    if (!aligned(x, 2 * esz) || !aligned(y, 2 * esz) || (x2 && !aligned(x2, 2 * esz)) || !aligned(g, 8))
        return set_error(HY_ERR_INVALID_ARG, "spectral_gate: misaligned pointer");
    if (overlap(x, nbytes, y, nbytes) || overlap(x2, nbytes, y, nbytes))
        return set_error(HY_ERR_INVALID_ARG, "spectral_gate: y aliases an input");
    const int64_t rows = (int64_t)B * H * Dh;
    if (rows > 0x7fffffffLL) return set_error(HY_ERR_UNSUPPORTED, "spectral_gate: too many rows");
    hy_status st = prologue((cudaStream_t)stream);
    if (st != HY_OK) return st;
    const int M = L / 2;
    ResidentParams p{};
    p.n_rows = rows;
    p.L = L;
    p.K = 1;
    p.B = 1;
    p.D = 1;
    p.remap = 0;
    p.u = x;
    p.gate[0] = x2;
    p.spec[0] = reinterpret_cast<const float2 *>(g);
    p.skip[0] = nullptr;
    p.spec_row_stride = M + 1;
    p.sdiv = Dh;
    p.smod = H;
    p.spec_batch_stride = g_batch_stride;
    p.y = y;
    p.scale = (float)(1.0 / (2.0 * (double)L));
    return launch_resident_conv(p, ilog2(M), dt, true, (cudaStream_t)stream);
}

}  // extern "C"

// ----------------------------------------------------------------------------
// hyena_operator_noalloc: the operator for callers that cannot allocate device
// memory (see include/hyena.h).  Sequences that fit on chip run exactly as in
// hyena_operator; longer ones use the multi-pass kernels with their workspace
// in the library's static device scratch instead of a caller buffer.
// ----------------------------------------------------------------------------
extern "C" hy_status hyena_operator_noalloc(int order, int B, int D, int L, hy_dtype dt, const void *v,
                                            const void *const *x, const hy_c32 *const *H,
                                            const float *const *Dskip, void *y, void *stream) {
    clear_error();
    const char *who = "hyena_operator_noalloc";
    if (order < 2 || order - 1 > kMaxOrders)
        return set_error(HY_ERR_UNSUPPORTED, "%s: order must be 2..%d", who, kMaxOrders + 1);
    if (!x || !H) return set_error(HY_ERR_INVALID_ARG, "%s: null x or H array", who);
    const int K = order - 1;
    for (int k = 0; k < K; ++k)
        if (!x[k]) return set_error(HY_ERR_INVALID_ARG, "%s: x[%d] is null", who, k);
    if (B < 1 || D < 1 || L < 1) return set_error(HY_ERR_INVALID_ARG, "%s: B, D, L must be >= 1", who);
    if (dt != HY_F32 && dt != HY_BF16) return set_error(HY_ERR_INVALID_ARG, "%s: unknown dtype", who);
    if (!v || !y) return set_error(HY_ERR_INVALID_ARG, "%s: null signal pointer", who);
    const size_t esz = dt_size(dt);
    const size_t nbytes = (size_t)B * D * L * esz;
    const size_t al = (L % 2 == 0) ? 2 * esz : esz;
    if (!aligned(v, al) || !aligned(y, al))
        return set_error(HY_ERR_INVALID_ARG, "%s: signals must be %zu-byte aligned", who, al);
    if (overlap(v, nbytes, y, nbytes)) return set_error(HY_ERR_INVALID_ARG, "%s: y aliases the input", who);
    const int64_t M = spectrum_m(L);
    for (int k = 0; k < K; ++k) {
        if (!H[k] || !aligned(H[k], 8)) return set_error(HY_ERR_INVALID_ARG, "%s: spectrum %d null or misaligned", who, k);
        if (!aligned(x[k], al)) return set_error(HY_ERR_INVALID_ARG, "%s: gate %d misaligned", who, k);
        if (overlap(x[k], nbytes, y, nbytes)) return set_error(HY_ERR_INVALID_ARG, "%s: y aliases gate %d", who, k);
    }
    const int log_m = ilog2(M);
    if (log_m <= kMaxResidentLogM) {
        // on chip: no workspace of any kind
        const void *no_ws = nullptr;
        return run_chain(K, B, D, L, dt, v, x, H, Dskip, y, const_cast<void *>(no_ws), 0,
                         (cudaStream_t)stream, who);
    }
    // one row's intermediates (8 bytes per complex point) must fit the scratch
    if ((size_t)8 * (size_t)M > noalloc_scratch_bytes())
        return set_error(HY_ERR_WORKSPACE, "%s: L=%d needs %zu scratch bytes per row; the static scratch holds %zu",
                         who, L, (size_t)8 * (size_t)M, noalloc_scratch_bytes());
    if (log_m > 20) return set_error(HY_ERR_UNSUPPORTED, "%s: L=%d is beyond the supported length", who, L);
    hy_status st = prologue((cudaStream_t)stream);
    if (st != HY_OK) return st;
    LongConvArgs a{};
    a.K = K;
    a.B = B;
    a.D = D;
    a.L = L;
    a.log_mc = log_m;
    a.dt = dt;
    a.u = v;
    for (int k = 0; k < K; ++k) {
        a.gate[k] = x[k];
        a.spec[k] = reinterpret_cast<const float2 *>(H[k]);
        a.skip[k] = Dskip ? Dskip[k] : nullptr;
    }
    a.y = y;
    return launch_long_conv_noalloc(a, (cudaStream_t)stream);
}

// ----------------------------------------------------------------------------
// Host-buffer entry points (see include/hyena.h and host_pipeline.h): the
// operator and the spectral gate over signals in host memory, with the
// host-to-device copies, the compute and the device-to-host copies of
// successive row chunks overlapped.
// ----------------------------------------------------------------------------
namespace {

// Chunks of a (B, G, row) signal: whole batches when one batch is at most the
// target size, else runs of `ng` groups (channels or heads) within one batch.
struct HostPlan {
    bool whole;       // chunks are nb whole batches
    int nb, ng;       // batches per chunk (whole) or groups per chunk
    int per_batch;    // chunks per batch (!whole)
    int nchunks;
    int64_t max_groups;   // groups in the largest chunk
};

HostPlan host_plan(int B, int G, size_t group_bytes, int min_groups) {
    HostPlan p{};
    int64_t g = (int64_t)(kHostChunkBytes / (group_bytes ? group_bytes : 1));
    if (g < min_groups) g = min_groups;
    if (g < 1) g = 1;
    if (g >= G) {
        p.whole = true;
        p.nb = (int)((g / G) < B ? (g / G) : B);
        if (p.nb < 1) p.nb = 1;
        p.ng = G;
        p.nchunks = (B + p.nb - 1) / p.nb;
        p.max_groups = (int64_t)p.nb * G;
    } else {
        p.whole = false;
        p.nb = 1;
        p.ng = (int)g;
        p.per_batch = (G + p.ng - 1) / p.ng;
        p.nchunks = B * p.per_batch;
        p.max_groups = p.ng;
    }
    return p;
}

// chunk c of plan p: first batch b0, batches nbc, first group g0, groups ngc
void host_chunk(const HostPlan &p, int B, int G, int c, int &b0, int &nbc, int &g0, int &ngc) {
    if (p.whole) {
        b0 = c * p.nb;
        nbc = (B - b0) < p.nb ? (B - b0) : p.nb;
        g0 = 0;
        ngc = G;
    } else {
        b0 = c / p.per_batch;
        nbc = 1;
        g0 = (c % p.per_batch) * p.ng;
        ngc = (G - g0) < p.ng ? (G - g0) : p.ng;
    }
}

size_t host_ring_bytes(int n_in, size_t slot) { return (size_t)kHostSlots * ((size_t)n_in * round256(slot) + round256(slot)); }

HostPlan operator_host_plan(int D, int B, int L, hy_dtype dt) {
    const int log_m = ilog2(spectrum_m(L));
    // multi-pass chunks of at least 8 rows keep its launches full
    return host_plan(B, D, (size_t)L * dt_size(dt), log_m > kMaxResidentLogM ? 8 : 1);
}

}  // namespace

extern "C" size_t hyena_operator_host_workspace(int order, int B, int D, int L, hy_dtype dt) {
    if (order < 2 || order - 1 > kMaxOrders || B < 1 || D < 1 || L < 1 || (dt != HY_F32 && dt != HY_BF16)) return 0;
    const HostPlan p = operator_host_plan(D, B, L, dt);
    const size_t slot = (size_t)p.max_groups * L * dt_size(dt);
    const size_t chain = hyena_operator_workspace(order, 1, (int)p.max_groups, L, dt);
    return host_ring_bytes(order, slot) + round256(chain);
}

extern "C" hy_status hyena_operator_host(int order, int B, int D, int L, hy_dtype dt, const void *v,
                                         const void *const *x, const hy_c32 *const *H,
                                         const float *const *Dskip, void *y, void *ws, size_t ws_bytes,
                                         void *stream) {
    clear_error();
    const char *who = "hyena_operator_host";
    if (order < 2 || order - 1 > kMaxOrders)
        return set_error(HY_ERR_UNSUPPORTED, "%s: order must be 2..%d", who, kMaxOrders + 1);
    if (B < 1 || D < 1 || L < 1) return set_error(HY_ERR_INVALID_ARG, "%s: B, D, L must be >= 1", who);
    if (dt != HY_F32 && dt != HY_BF16) return set_error(HY_ERR_INVALID_ARG, "%s: unknown dtype", who);
    if (!x || !H) return set_error(HY_ERR_INVALID_ARG, "%s: null x or H array", who);
    const int K = order - 1;
    hy_status st;
    if ((st = check_host_ptr(v, who, "v")) != HY_OK || (st = check_host_ptr(y, who, "y")) != HY_OK) return st;
    for (int k = 0; k < K; ++k) {
        if ((st = check_host_ptr(x[k], who, "x[k]")) != HY_OK) return st;
        if (!H[k]) return set_error(HY_ERR_INVALID_ARG, "%s: H[%d] is null", who, k);
    }
    const size_t need = hyena_operator_host_workspace(order, B, D, L, dt);
    if (!ws || ws_bytes < need)
        return set_error(HY_ERR_WORKSPACE, "%s: needs %zu workspace bytes, got %zu", who, need, ws ? ws_bytes : (size_t)0);
    if (!aligned(ws, 256)) return set_error(HY_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
    const size_t esz = dt_size(dt);
    const HostPlan p = operator_host_plan(D, B, L, dt);
    const size_t slot = (size_t)p.max_groups * L * esz;
    char *ring = reinterpret_cast<char *>(ws);
    char *chain_ws = ring + host_ring_bytes(order, slot);
    const size_t chain_bytes = ws_bytes - host_ring_bytes(order, slot);
    const int64_t M = spectrum_m(L);
    auto describe = [&](int c, HostChunk &ch) {
        int b0, nbc, g0, ngc;
        host_chunk(p, B, D, c, b0, nbc, g0, ngc);
        const size_t off = ((size_t)b0 * D + g0) * L * esz;
        ch.in_bytes = (size_t)nbc * ngc * L * esz;
        ch.src[0] = reinterpret_cast<const char *>(v) + off;
        for (int k = 0; k < K; ++k) ch.src[1 + k] = reinterpret_cast<const char *>(x[k]) + off;
        ch.dst = reinterpret_cast<char *>(y) + off;
        ch.out_bytes = ch.in_bytes;
    };
    auto compute = [&](int c, const void *const *din, void *dout, cudaStream_t s) {
        int b0, nbc, g0, ngc;
        host_chunk(p, B, D, c, b0, nbc, g0, ngc);
        const hy_c32 *Hc[kMaxOrders];
        const float *Dc[kMaxOrders];
        for (int k = 0; k < K; ++k) {
            Hc[k] = H[k] + (size_t)g0 * (M + 1);
            Dc[k] = (Dskip && Dskip[k]) ? Dskip[k] + g0 : nullptr;
        }
        return run_chain(K, nbc, ngc, L, dt, din[0], din + 1, Hc, Dskip ? Dc : nullptr, dout, chain_ws,
                         chain_bytes, s, who);
    };
    return run_host_pipeline(order, p.nchunks, slot, slot, ring, (cudaStream_t)stream, describe, compute, who);
}

extern "C" size_t spectral_gate_host_workspace(int B, int H, int Dh, int L, hy_dtype dt) {
    if (B < 1 || H < 1 || Dh < 1 || L < 1 || (dt != HY_F32 && dt != HY_BF16)) return 0;
    const HostPlan p = host_plan(B, H, (size_t)Dh * L * dt_size(dt), 1);
    return host_ring_bytes(2, (size_t)p.max_groups * Dh * L * dt_size(dt));
}

extern "C" hy_status spectral_gate_host(int B, int H, int Dh, int L, hy_dtype dt, const void *x, const hy_c32 *g,
                                        int64_t g_batch_stride, const void *x2, void *y, void *ws, size_t ws_bytes,
                                        void *stream) {
    clear_error();
    const char *who = "spectral_gate_host";
    if (B < 1 || H < 1 || Dh < 1 || L < 1) return set_error(HY_ERR_INVALID_ARG, "%s: B, H, Dh, L must be >= 1", who);
    if (dt != HY_F32 && dt != HY_BF16) return set_error(HY_ERR_INVALID_ARG, "%s: unknown dtype", who);
    if (!g) return set_error(HY_ERR_INVALID_ARG, "%s: null gate", who);
    if (g_batch_stride < 0) return set_error(HY_ERR_INVALID_ARG, "%s: negative gate stride", who);
    hy_status st;
    if ((st = check_host_ptr(x, who, "x")) != HY_OK || (st = check_host_ptr(y, who, "y")) != HY_OK) return st;
    if (x2 && (st = check_host_ptr(x2, who, "x2")) != HY_OK) return st;
    const size_t need = spectral_gate_host_workspace(B, H, Dh, L, dt);
    if (!ws || ws_bytes < need)
        return set_error(HY_ERR_WORKSPACE, "%s: needs %zu workspace bytes, got %zu", who, need, ws ? ws_bytes : (size_t)0);
    if (!aligned(ws, 256)) return set_error(HY_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
    const size_t esz = dt_size(dt);
    const HostPlan p = host_plan(B, H, (size_t)Dh * L * esz, 1);
    const size_t slot = (size_t)p.max_groups * Dh * L * esz;
    const int n_in = x2 ? 2 : 1;
    const int64_t nbins = L / 2 + 1;
    auto describe = [&](int c, HostChunk &ch) {
        int b0, nbc, h0, nhc;
        host_chunk(p, B, H, c, b0, nbc, h0, nhc);
        const size_t off = (((size_t)b0 * H + h0) * Dh) * L * esz;
        ch.in_bytes = (size_t)nbc * nhc * Dh * L * esz;
        ch.src[0] = reinterpret_cast<const char *>(x) + off;
        if (x2) ch.src[1] = reinterpret_cast<const char *>(x2) + off;
        ch.dst = reinterpret_cast<char *>(y) + off;
        ch.out_bytes = ch.in_bytes;
    };
    auto compute = [&](int c, const void *const *din, void *dout, cudaStream_t s) {
        int b0, nbc, h0, nhc;
        host_chunk(p, B, H, c, b0, nbc, h0, nhc);
        const hy_c32 *gc = g + (size_t)b0 * g_batch_stride + (size_t)h0 * nbins;
        return spectral_gate(nbc, nhc, Dh, L, dt, din[0], gc, g_batch_stride, x2 ? din[1] : nullptr, dout, s);
    };
    return run_host_pipeline(n_in, p.nchunks, slot, slot, reinterpret_cast<char *>(ws), (cudaStream_t)stream,
                             describe, compute, who);
}

extern "C" size_t hyena_nd_conv_host_workspace(int ndim, const int *dims, int B, int D, int circular) {
    if (ndim != 3 || !dims || B < 1 || D < 1 || dims[0] < 1 || dims[1] < 1 || dims[2] < 1) return 0;
    const size_t vox = (size_t)dims[0] * dims[1] * dims[2];
    const HostPlan p = host_plan(B, D, vox * 4, 1);
    const size_t chain = hyena_nd_conv_workspace(ndim, dims, 1, (int)p.max_groups, circular);
    return host_ring_bytes(2, (size_t)p.max_groups * vox * 4) + round256(chain);
}

extern "C" hy_status hyena_nd_conv_host(int ndim, const int *dims, int B, int D, int circular, const float *u,
                                        const hy_c32 *H, int64_t H_batch_stride, const float *Dskip,
                                        const float *gate, float *y, void *ws, size_t ws_bytes, void *stream) {
    clear_error();
    const char *who = "hyena_nd_conv_host";
    if (ndim != 3) return set_error(HY_ERR_UNSUPPORTED, "%s: only ndim = 3 is built", who);
    if (!dims || !H) return set_error(HY_ERR_INVALID_ARG, "%s: null pointer", who);
    if (B < 1 || D < 1 || H_batch_stride < 0) return set_error(HY_ERR_INVALID_ARG, "%s: bad B, D or stride", who);
    for (int i = 0; i < 3; ++i)
        if (dims[i] < 1) return set_error(HY_ERR_INVALID_ARG, "%s: bad grid", who);
    hy_status st;
    if ((st = check_host_ptr(u, who, "u")) != HY_OK || (st = check_host_ptr(y, who, "y")) != HY_OK) return st;
    if (gate && (st = check_host_ptr(gate, who, "gate")) != HY_OK) return st;
    const size_t need = hyena_nd_conv_host_workspace(ndim, dims, B, D, circular);
    if (!ws || ws_bytes < need)
        return set_error(HY_ERR_WORKSPACE, "%s: needs %zu workspace bytes, got %zu", who, need, ws ? ws_bytes : (size_t)0);
    if (!aligned(ws, 256)) return set_error(HY_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
    const size_t vox = (size_t)dims[0] * dims[1] * dims[2];
    const HostPlan p = host_plan(B, D, vox * 4, 1);
    const size_t slot = (size_t)p.max_groups * vox * 4;
    const int n_in = gate ? 2 : 1;
    char *ring = reinterpret_cast<char *>(ws);
    char *chain_ws = ring + host_ring_bytes(2, slot);
    const size_t chain_bytes = ws_bytes - host_ring_bytes(2, slot);
    int S[3];
    for (int i = 0; i < 3; ++i) S[i] = circular ? dims[i] : 2 * dims[i];
    const size_t spec_per_channel = (size_t)S[0] * S[1] * (S[2] / 2 + 1);
    auto describe = [&](int c, HostChunk &ch) {
        int b0, nbc, d0, ndc;
        host_chunk(p, B, D, c, b0, nbc, d0, ndc);
        const size_t off = ((size_t)b0 * D + d0) * vox;
        ch.in_bytes = (size_t)nbc * ndc * vox * 4;
        ch.src[0] = u + off;
        if (gate) ch.src[1] = gate + off;
        ch.dst = y + off;
        ch.out_bytes = ch.in_bytes;
    };
    auto compute = [&](int c, const void *const *din, void *dout, cudaStream_t s) {
        int b0, nbc, d0, ndc;
        host_chunk(p, B, D, c, b0, nbc, d0, ndc);
        const hy_c32 *Hc = H + (size_t)b0 * H_batch_stride + (size_t)d0 * spec_per_channel;
        return hyena_nd_conv(ndim, dims, nbc, ndc, circular, reinterpret_cast<const float *>(din[0]), Hc,
                             H_batch_stride, Dskip ? Dskip + d0 : nullptr,
                             gate ? reinterpret_cast<const float *>(din[1]) : nullptr,
                             reinterpret_cast<float *>(dout), chain_bytes ? chain_ws : nullptr, chain_bytes, s);
    };
    return run_host_pipeline(n_in, p.nchunks, slot, slot, ring, (cudaStream_t)stream, describe, compute, who);
}

// ----------------------------------------------------------------------------
// Backward pass of the 1-D operator (see include/hyena.h and backward.cu):
// forward recompute, then per order from the last: dx_k, the reversed e_k,
// dD_k, dh_k (a convolution of z_{k-1} with per-row spectra of the reversed
// e_k, summed over the batch) and the next gradient (a convolution of the
// reversed e_k with h_k, read back reversed, plus D_k e_k).  Every
// convolution is the forward path's (run_chain); intermediates are fp32 rows
// in the workspace.
// ----------------------------------------------------------------------------
namespace {

struct BwLayout {
    size_t row;            // bytes of one fp32 signal (all rows)
    size_t c, z, g, er, r, w, es, chain;   // offsets
    size_t chain_bytes, total;
};

BwLayout bw_layout(int K, int B, int D, int L) {
    BwLayout p{};
    const int64_t R = (int64_t)B * D;
    const int64_t M = spectrum_m(L);
    p.row = round256((size_t)R * L * 4);
    size_t o = 0;
    p.c = o; o += (size_t)K * p.row;
    p.z = o; o += (size_t)K * p.row;
    p.g = o; o += p.row;
    p.er = o; o += p.row;
    p.r = o; o += p.row;
    p.w = o; o += p.row;
    p.es = o; o += round256((size_t)R * (M + 1) * 8);
    const int Lc = L;
    size_t ch = hyena_operator_workspace(2, B, D, L, HY_F32);
    const size_t ch2 = hyena_operator_workspace(2, 1, (int)R, L, HY_F32);
    const size_t ch3 = hyena_filter_spectrum_workspace(R, 1, &Lc, 0);
    ch = ch > ch2 ? ch : ch2;
    ch = ch > ch3 ? ch : ch3;
    p.chain = o;
    p.chain_bytes = round256(ch);
    o += p.chain_bytes;
    p.total = o;
    return p;
}

}  // namespace

extern "C" size_t hyena_operator_backward_workspace(int order, int B, int D, int L, hy_dtype dt) {
    if (order < 2 || order - 1 > kMaxOrders || B < 1 || D < 1 || L < 1 || (dt != HY_F32 && dt != HY_BF16)) return 0;
    if ((int64_t)B * D > 0x7fffffffLL) return 0;
    return bw_layout(order - 1, B, D, L).total;
}

extern "C" hy_status hyena_operator_backward(int order, int B, int D, int L, hy_dtype dt, const void *v,
                                             const void *const *x, const hy_c32 *const *H,
                                             const float *const *Dskip, const void *dy, void *dv,
                                             void *const *dx, float *const *dh, float *const *dD, void *ws,
                                             size_t ws_bytes, void *stream) {
    clear_error();
    const char *who = "hyena_operator_backward";
    if (order < 2 || order - 1 > kMaxOrders)
        return set_error(HY_ERR_UNSUPPORTED, "%s: order must be 2..%d", who, kMaxOrders + 1);
    if (B < 1 || D < 1 || L < 1) return set_error(HY_ERR_INVALID_ARG, "%s: B, D, L must be >= 1", who);
    if (dt != HY_F32 && dt != HY_BF16) return set_error(HY_ERR_INVALID_ARG, "%s: unknown dtype", who);
    if (!v || !dy || !dv || !x || !H || !dx) return set_error(HY_ERR_INVALID_ARG, "%s: null pointer", who);
    const int K = order - 1;
    const size_t esz = dt_size(dt);
    const size_t al = (L % 2 == 0) ? 2 * esz : esz;
    if (!aligned(v, al) || !aligned(dy, al) || !aligned(dv, al))
        return set_error(HY_ERR_INVALID_ARG, "%s: signals must be %zu-byte aligned", who, al);
    for (int k = 0; k < K; ++k) {
        if (!x[k] || !H[k] || !dx[k]) return set_error(HY_ERR_INVALID_ARG, "%s: null x, H or dx of order %d", who, k);
        if (!aligned(x[k], al) || !aligned(dx[k], al) || !aligned(H[k], 8))
            return set_error(HY_ERR_INVALID_ARG, "%s: order %d misaligned", who, k);
    }
    if ((int64_t)B * D > 0x7fffffffLL) return set_error(HY_ERR_UNSUPPORTED, "%s: too many rows", who);
    const BwLayout lay = bw_layout(K, B, D, L);
    if (!ws || ws_bytes < lay.total)
        return set_error(HY_ERR_WORKSPACE, "%s: needs %zu workspace bytes, got %zu", who, lay.total, ws ? ws_bytes : (size_t)0);
    if (!aligned(ws, 256)) return set_error(HY_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
    cudaStream_t s = (cudaStream_t)stream;
    // order 2 over power-of-two rows that fit on chip: one fused kernel
    // (both transforms of every row and the batch sums of dh and dD on chip)
    {
        const void *p16[5] = {v, x[0], dy, dv, dx[0]};
        float *dh0 = dh ? dh[0] : nullptr;
        float *dD0 = dD ? dD[0] : nullptr;
        if (bw_fused_eligible(order, L, dt, p16, 5) && (!dh0 || aligned(dh0, 8))) {
            hy_status st = prologue(s);
            if (st != HY_OK) return st;
            return launch_bw_fused(B, D, L, dt, v, x[0], dy, H[0], Dskip ? Dskip[0] : nullptr, dv, dx[0], dh0, dD0, s);
        }
    }
    char *base = reinterpret_cast<char *>(ws);
    auto buf = [&](size_t off) { return reinterpret_cast<float *>(base + off); };
    float *c[kMaxOrders], *z[kMaxOrders];
    for (int k = 0; k < K; ++k) {
        c[k] = buf(lay.c + (size_t)k * lay.row);
        z[k] = buf(lay.z + (size_t)k * lay.row);
    }
    float *g = buf(lay.g), *er = buf(lay.er), *r = buf(lay.r), *w = buf(lay.w);
    hy_c32 *es = reinterpret_cast<hy_c32 *>(base + lay.es);
    void *chain = base + lay.chain;
    const int64_t R = (int64_t)B * D;
    const int64_t n = R * L;
    hy_status st = prologue(s);
    if (st != HY_OK) return st;
    // ---- forward recompute: z_0 = v; c_k = h_k * z_{k-1} + D_k z_{k-1}; z_k = x_k ⊙ c_k
    if ((st = bw_to_f32(v, dt, z[0], n, s)) != HY_OK) return st;
    for (int k = 0; k < K; ++k) {
        const void *nog[1] = {nullptr};
        const hy_c32 *Hk[1] = {H[k]};
        const float *Sk[1] = {Dskip ? Dskip[k] : nullptr};
        if ((st = run_chain(1, B, D, L, HY_F32, z[k], nog, Hk, Sk, c[k], chain, lay.chain_bytes, s, who)) != HY_OK)
            return st;
        if (k + 1 < K && (st = bw_gate(x[k], dt, c[k], z[k + 1], n, s)) != HY_OK) return st;
    }
    // ---- backward from the last order
    if ((st = bw_to_f32(dy, dt, g, n, s)) != HY_OK) return st;
    for (int k = K - 1; k >= 0; --k) {
        if (dD && dD[k] && (st = bw_dD(g, x[k], dt, z[k], dD[k], B, D, L, s)) != HY_OK) return st;
        if ((st = bw_dx_e(g, c[k], x[k], dt, dx[k], er, R, L, s)) != HY_OK) return st;
        const void *nog[1] = {nullptr};
        const float *nos[1] = {nullptr};
        if (dh && dh[k]) {
            // w = z_{k-1} * reverse(e_k) with each row's own spectrum, then
            // dh_k[d][τ] = Σ_b w[b, d][L-1-τ]
            const int Lr = L;
            if ((st = hyena_filter_spectrum(R, 1, &Lr, 0, er, es, chain, lay.chain_bytes, s)) != HY_OK) return st;
            const hy_c32 *Es[1] = {es};
            if ((st = run_chain(1, 1, (int)R, L, HY_F32, z[k], nog, Es, nos, w, chain, lay.chain_bytes, s, who)) != HY_OK)
                return st;
            if ((st = bw_dh(w, dh[k], B, D, L, s)) != HY_OK) return st;
        }
        // g_{k-1}[s] = (h_k * reverse(e_k))[L-1-s] + D_k e_k[s]
        const hy_c32 *Hk[1] = {H[k]};
        if ((st = run_chain(1, B, D, L, HY_F32, er, nog, Hk, nos, r, chain, lay.chain_bytes, s, who)) != HY_OK)
            return st;
        if ((st = bw_next_g(r, g, x[k], dt, Dskip ? Dskip[k] : nullptr, R, D, L, s)) != HY_OK) return st;
    }
    return bw_from_f32(g, dt, dv, n, s);
}

extern "C" hy_status spectral_gate_decode(int B, int H, int Dh, int n, hy_dtype dt, int64_t pos, const void *x,
                                          const hy_c32 *g, int64_t g_batch_stride, const void *x2, hy_c32 *cache,
                                          void *y, void *stream) {
    clear_error();
    const char *who = "spectral_gate_decode";
    if (B < 1 || H < 1 || Dh < 1) return set_error(HY_ERR_INVALID_ARG, "%s: B, H, Dh must be >= 1", who);
    if (dt != HY_F32 && dt != HY_BF16) return set_error(HY_ERR_INVALID_ARG, "%s: unknown dtype", who);
    if (!is_pow2(n) || n < 2 || n > (1 << 24))
        return set_error(HY_ERR_UNSUPPORTED, "%s: n must be a power of two in [2, 2^24]", who);
    if (pos < 0 || pos >= n) return set_error(HY_ERR_INVALID_ARG, "%s: pos %lld outside [0, %d)", who, (long long)pos, n);
    if (!x || !g || !cache || !y) return set_error(HY_ERR_INVALID_ARG, "%s: null pointer", who);
    if (g_batch_stride < 0) return set_error(HY_ERR_INVALID_ARG, "%s: negative gate stride", who);
    if (!aligned(g, 8) || !aligned(cache, 8)) return set_error(HY_ERR_INVALID_ARG, "%s: g and cache must be 8-byte aligned", who);
    const int64_t rows = (int64_t)B * H * Dh;
    const size_t esz = dt_size(dt);
    if (overlap(cache, (size_t)rows * (n / 2 + 1) * 8, y, (size_t)rows * esz) ||
        overlap(x, (size_t)rows * esz, y, (size_t)rows * esz))
        return set_error(HY_ERR_INVALID_ARG, "%s: y aliases an input", who);
    GateDecodeArgs a{};
    a.rows = rows;
    a.n = n;
    a.pos = pos;
    a.dh = Dh;
    a.heads = H;
    a.g = reinterpret_cast<const float2 *>(g);
    a.g_batch_stride = g_batch_stride;
    a.cache = reinterpret_cast<float2 *>(cache);
    return launch_gate_decode(a, dt, x, x2, y, (cudaStream_t)stream);
}
