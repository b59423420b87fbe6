// C ABI of libgdn2: argument validation on the host, then kernel dispatch on the
// caller's stream.  Nothing here allocates device memory.
#include <stdio.h>
#include <string.h>

#include "common.cuh"

namespace gdn2 {
void set_wait_limit(long long cycles);
cudaError_t read_device_error(unsigned int *value, bool clear);
}  // namespace gdn2

namespace {

thread_local char g_last_error[256] = "";

gdn2_status fail(gdn2_status s, const char *fmt, const char *detail) {
    snprintf(g_last_error, sizeof(g_last_error), fmt, detail);
    return s;
}

gdn2_status cuda_status(cudaError_t err, const char *where) {
    if (err == cudaSuccess) return GDN2_OK;
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(err));
    return GDN2_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gdn2_status check_common(int B, int H, int dk, int dv, gdn2_dtype dt) {
    if (B < 0 || H < 0) return fail(GDN2_ERR_INVALID_ARG, "%s", "negative B or H");
    if (dt != GDN2_BF16 && dt != GDN2_FP32) return fail(GDN2_ERR_UNSUPPORTED, "%s", "unknown dtype");
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128))
        return fail(GDN2_ERR_UNSUPPORTED, "%s", "head sizes must be 64 or 128");
    return GDN2_OK;
}

gdn2_status check_ptr(const void *p, const char *name) {
    if (!p) return fail(GDN2_ERR_INVALID_ARG, "null pointer: %s", name);
    if (!aligned16(p)) return fail(GDN2_ERR_INVALID_ARG, "pointer not 16-byte aligned: %s", name);
    return GDN2_OK;
}

// [a, a+na) and [b, b+nb) overlap?
bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const char *pa = static_cast<const char *>(a), *pb = static_cast<const char *>(b);
    return pa < pb + nb && pb < pa + na;
}

}  // namespace

namespace gdn2 {
// The message gdn2_last_error() returns on this thread, for entry points defined
// in other files of the library.
void set_last_error(const char *message) { snprintf(g_last_error, sizeof(g_last_error), "%s", message); }
}  // namespace gdn2

extern "C" {

const char *gdn2_status_string(gdn2_status s) {
    switch (s) {
        case GDN2_OK: return "GDN2_OK";
        case GDN2_ERR_INVALID_ARG: return "GDN2_ERR_INVALID_ARG";
        case GDN2_ERR_UNSUPPORTED: return "GDN2_ERR_UNSUPPORTED";
        case GDN2_ERR_CUDA: return "GDN2_ERR_CUDA";
    }
    return "GDN2_UNKNOWN_STATUS";
}

const char *gdn2_last_error(void) { return g_last_error; }

int gdn2_version(void) { return 200; }

gdn2_status gdn2_set_wait_limit(long long cycles) {
    gdn2::set_wait_limit(cycles > 0 ? cycles : 4000000000ll);
    return GDN2_OK;
}

gdn2_status gdn2_device_error(unsigned int *code, int clear) {
    if (!code) return fail(GDN2_ERR_INVALID_ARG, "%s", "null pointer: code");
    return cuda_status(gdn2::read_device_error(code, clear != 0), "gdn2_device_error");
}

// Shared host-side checks and dispatch of the two prefill entry points.  nseq
// sequences of T tokens each (cu == nullptr), or nseq packed sequences whose
// device offsets cu[0..nseq] index T tokens in all.
static gdn2_status chunk_fwd_common(const void *q, const void *k, const void *v, const float *alpha,
                                    const float *b, const float *w, const int *cu, const float *S0, void *o,
                                    float *S_T, int nseq, int T, int H, int d_k, int d_v, gdn2_dtype dt,
                                    void *stream, bool launch = true) {
    g_last_error[0] = 0;
    gdn2_status st = check_common(nseq, H, d_k, d_v, dt);
    if (st != GDN2_OK) return st;
    if (T < 0) return fail(GDN2_ERR_INVALID_ARG, "%s", "negative T");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (nseq == 0 || H == 0) return GDN2_OK;
    const size_t es = dt == GDN2_BF16 ? 2 : 4;
    const size_t state_bytes = (size_t)nseq * H * d_k * d_v * sizeof(float);
    if (S0 && (st = check_ptr(S0, "S0")) != GDN2_OK) return st;
    if (S_T && (st = check_ptr(S_T, "S_T")) != GDN2_OK) return st;
    if (S0 && S_T && S0 != S_T && overlaps(S0, state_bytes, S_T, state_bytes))
        return fail(GDN2_ERR_INVALID_ARG, "%s", "S_T partially overlaps S0 (only exact aliasing is allowed)");
    if (cu) {
        if (reinterpret_cast<uintptr_t>(cu) & 3u) return fail(GDN2_ERR_INVALID_ARG, "%s", "cu_seqlens not 4-byte aligned");
    }
    if (T == 0) {          // every sequence is empty: S_T = S0
        if (!S_T || S_T == S0) return GDN2_OK;
        cudaError_t err = S0 ? cudaMemcpyAsync(S_T, S0, state_bytes, cudaMemcpyDeviceToDevice, s)
                             : cudaMemsetAsync(S_T, 0, state_bytes, s);
        return cuda_status(err, "T = 0 state copy");
    }
    const void *ins[6] = {q, k, v, alpha, b, w};
    const char *names[6] = {"q", "k", "v", "alpha", "b", "w"};
    for (int i = 0; i < 6; ++i)
        if ((st = check_ptr(ins[i], names[i])) != GDN2_OK) return st;
    if ((st = check_ptr(o, "o")) != GDN2_OK) return st;
    const size_t tok = (size_t)(cu ? 1 : nseq) * T * H;
    const size_t in_bytes[6] = {tok * d_k * es, tok * d_k * es, tok * d_v * es,
                                tok * d_k * 4,  tok * d_k * 4,  tok * d_v * 4};
    const size_t o_bytes = tok * d_v * es;
    for (int i = 0; i < 6; ++i)
        if (overlaps(o, o_bytes, ins[i], in_bytes[i])) return fail(GDN2_ERR_INVALID_ARG, "o overlaps %s", names[i]);
    if (overlaps(o, o_bytes, S0, state_bytes) || overlaps(o, o_bytes, S_T, state_bytes))
        return fail(GDN2_ERR_INVALID_ARG, "%s", "o overlaps a state buffer");
    if (S_T)
        for (int i = 0; i < 6; ++i)
            if (overlaps(S_T, state_bytes, ins[i], in_bytes[i]))
                return fail(GDN2_ERR_INVALID_ARG, "S_T overlaps %s", names[i]);
    if (cu) {
        const size_t cu_bytes = (size_t)(nseq + 1) * sizeof(int);
        if (overlaps(o, o_bytes, cu, cu_bytes) || overlaps(S_T, state_bytes, cu, cu_bytes))
            return fail(GDN2_ERR_INVALID_ARG, "%s", "an output overlaps cu_seqlens");
    }

    if (!launch) return GDN2_OK;
    cudaError_t err;
    if (gdn2::chunk_tc_supported(d_k, d_v, dt))
        err = gdn2::launch_chunk_tc(q, k, v, alpha, b, w, S0, o, S_T, nseq, T, H, cu, false, s);
    else
        err = gdn2::launch_chunk_simt(q, k, v, alpha, b, w, S0, o, S_T, nseq, T, H, d_k, d_v, dt, cu, s);
    return cuda_status(err, "gdn2_chunk_fwd launch");
}

gdn2_status gdn2_chunk_fwd(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                           const float *w, const float *S0, void *o, float *S_T, int B, int T, int H, int d_k,
                           int d_v, gdn2_dtype dt, void *stream) {
    return chunk_fwd_common(q, k, v, alpha, b, w, nullptr, S0, o, S_T, B, T, H, d_k, d_v, dt, stream);
}

gdn2_status gdn2_chunk_fwd_varlen(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                                  const float *w, const int32_t *cu_seqlens, int N, const float *S0, void *o,
                                  float *S_T, int T_total, int H, int d_k, int d_v, gdn2_dtype dt, void *stream) {
    g_last_error[0] = 0;
    if (!cu_seqlens && N > 0) return fail(GDN2_ERR_INVALID_ARG, "%s", "null pointer: cu_seqlens");
    return chunk_fwd_common(q, k, v, alpha, b, w, reinterpret_cast<const int *>(cu_seqlens), S0, o, S_T, N, T_total,
                            H, d_k, d_v, dt, stream);
}

}  // extern "C"

namespace {
// Segments for gdn2_chunk_fwd_segmented: requested > 1 is capped at the number
// of 64-token chunks; 0 picks the count with the least estimated time, in
// chunk steps of one CTA per SM: 2 B H CTAs walk every chunk in one pass, or
// 4 B H (P - 1) and then 2 B H P CTAs walk ceil(chunks / P) chunks each, in
// waves of `sms` CTAs; each wave costs about 2 chunk steps more (start-up and
// drain) and each of the P - 1 combine steps about 1.3 (both measured on a
// B200 with the long workload, T = 65,573 and 16 heads, for P from 1 to 54).
// Segments are L = ceil(chunks / P) chunks long; P is then ceil(T / L).
void resolve_segments(int B, int T, int H, int d_k, int d_v, gdn2_dtype dt, int requested, int sms, int *P,
                      int *L) {
    *P = 1;
    *L = T;
    const long long nch = ((long long)T + 63) / 64;
    if (!gdn2::chunk_tc_supported(d_k, d_v, dt) || nch <= 1 || requested == 1 || B <= 0 || H <= 0) return;
    auto waves = [&](long long ctas) { return (ctas + sms - 1) / sms; };
    long long best_p = 1;
    if (requested > 1) {
        best_p = requested < nch ? requested : nch;
    } else {
        // tenths of a chunk step
        const long long bh = (long long)B * H, one = waves(2 * bh) * (nch + 2) * 10;
        long long best = one;
        for (long long p = 2; p <= 64 && p <= nch; ++p) {
            const long long cost =
                (waves(4 * bh * (p - 1)) + waves(2 * bh * p)) * ((nch + p - 1) / p + 2) * 10 + 13 * (p - 1);
            if (cost < best) {
                best = cost;
                best_p = p;
            }
        }
        if (best * 10 > one * 9) best_p = 1;     // not worth the three passes
    }
    if (best_p <= 1) return;
    const long long lc = (nch + best_p - 1) / best_p;
    *L = (int)(lc * 64);
    *P = (int)((T + *L - 1) / *L);
    if (*P <= 1) {
        *P = 1;
        *L = T;
    }
}

int current_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess || sms <= 0) {
        cudaGetLastError();
        return 0;
    }
    return sms;
}
}  // namespace

extern "C" {

size_t gdn2_chunk_fwd_segmented_workspace_size(int B, int T, int H, int d_k, int d_v, int segments) {
    if (B <= 0 || T <= 0 || H <= 0 || segments < 0) return 0;
    const int sms = segments == 0 ? current_sms() : 1;
    if (sms <= 0) return 0;
    int P = 1, L = T;
    resolve_segments(B, T, H, d_k, d_v, GDN2_BF16, segments, sms, &P, &L);
    return gdn2::segmented_workspace_bytes(B, H, P);
}

int gdn2_chunk_fwd_segments(int B, int T, int H, int d_k, int d_v, int segments) {
    if (B <= 0 || T <= 0 || H <= 0 || segments < 0) return 1;
    const int sms = segments == 0 ? current_sms() : 1;
    if (sms <= 0) return 1;
    int P = 1, L = T;
    resolve_segments(B, T, H, d_k, d_v, GDN2_BF16, segments, sms, &P, &L);
    return P;
}

gdn2_status gdn2_chunk_fwd_segmented(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                                     const float *w, const float *S0, void *o, float *S_T, int B, int T, int H,
                                     int d_k, int d_v, gdn2_dtype dt, int segments, void *workspace,
                                     size_t workspace_bytes, void *stream) {
    g_last_error[0] = 0;
    if (segments < 0) return fail(GDN2_ERR_INVALID_ARG, "%s", "negative segments");
    if (segments > 1 && !gdn2::chunk_tc_supported(d_k, d_v, dt))
        return fail(GDN2_ERR_UNSUPPORTED, "%s", "segments > 1 need BF16 q/k/v with d_k = d_v = 128");
    int P = 1, L = T;
    if (B > 0 && T > 0 && H > 0) {
        const int sms = segments == 0 ? current_sms() : 1;
        if (sms <= 0) return fail(GDN2_ERR_CUDA, "%s", "gdn2_chunk_fwd_segmented: no current CUDA device");
        resolve_segments(B, T, H, d_k, d_v, dt, segments, sms, &P, &L);
    }
    if (P <= 1) return gdn2_chunk_fwd(q, k, v, alpha, b, w, S0, o, S_T, B, T, H, d_k, d_v, dt, stream);
    gdn2_status st = chunk_fwd_common(q, k, v, alpha, b, w, nullptr, S0, o, S_T, B, T, H, d_k, d_v, dt, stream,
                                      false);
    if (st != GDN2_OK) return st;
    if ((long long)B * P > (1 << 20)) return fail(GDN2_ERR_UNSUPPORTED, "%s", "too many segments in all");
    if ((long long)B * T >= (1ll << 31)) return fail(GDN2_ERR_UNSUPPORTED, "%s", "B * T must be below 2^31");
    const size_t need = gdn2::segmented_workspace_bytes(B, H, P);
    if (!workspace) return fail(GDN2_ERR_INVALID_ARG, "%s", "null pointer: workspace");
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(GDN2_ERR_INVALID_ARG, "%s", "workspace not 256-byte aligned");
    if (workspace_bytes < need) {
        snprintf(g_last_error, sizeof(g_last_error),
                 "gdn2_chunk_fwd_segmented: workspace of %zu bytes, %zu needed for %d segments", workspace_bytes, need,
                 P);
        return GDN2_ERR_INVALID_ARG;
    }
    const size_t tok = (size_t)B * T * H, state_bytes = (size_t)B * H * d_k * d_v * sizeof(float);
    const void *bufs[9] = {q, k, v, alpha, b, w, o, S0, S_T};
    const char *names[9] = {"q", "k", "v", "alpha", "b", "w", "o", "S0", "S_T"};
    const size_t bytes[9] = {tok * d_k * 2, tok * d_k * 2, tok * d_v * 2, tok * d_k * 4, tok * d_k * 4,
                             tok * d_v * 4, tok * d_v * 2, state_bytes,   state_bytes};
    for (int i = 0; i < 9; ++i)
        if (overlaps(workspace, need, bufs[i], bytes[i])) return fail(GDN2_ERR_INVALID_ARG, "workspace overlaps %s", names[i]);
    cudaError_t err = gdn2::launch_chunk_segmented(q, k, v, alpha, b, w, S0, o, S_T, B, T, H, P, L, workspace,
                                                   static_cast<cudaStream_t>(stream));
    return cuda_status(err, "gdn2_chunk_fwd_segmented launch");
}

size_t gdn2_chunk_bwd_workspace_size(int B, int T, int H, int d_k, int d_v) {
    if (B < 0 || T < 0 || H < 0 || (d_k != 64 && d_k != 128) || (d_v != 64 && d_v != 128)) return 0;
    return gdn2::chunk_bwd_workspace_floats(B, T, H, d_k, d_v) * sizeof(float);
}

gdn2_status gdn2_chunk_bwd(const void *q, const void *k, const void *v, const float *alpha, const float *b,
                           const float *w, const float *S0, const void *dO, const float *dST, void *dq, void *dk,
                           void *dv, float *dalpha, float *db, float *dw, float *dS0, void *workspace,
                           size_t workspace_bytes, int B, int T, int H, int d_k, int d_v, gdn2_dtype dt,
                           void *stream) {
    g_last_error[0] = 0;
    gdn2_status st = check_common(B, H, d_k, d_v, dt);
    if (st != GDN2_OK) return st;
    if (T < 0) return fail(GDN2_ERR_INVALID_ARG, "%s", "negative T");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)B * H * d_k * d_v * sizeof(float);
    if (dS0 && (st = check_ptr(dS0, "dS0")) != GDN2_OK) return st;
    if (dST && (st = check_ptr(dST, "dST")) != GDN2_OK) return st;
    if (B == 0 || H == 0) return GDN2_OK;
    if ((long long)B * H > 65535)       // (sequence, head) pairs index the grid's second dimension
        return fail(GDN2_ERR_UNSUPPORTED, "%s", "gdn2_chunk_bwd: B * H above 65535");
    if (dS0 && overlaps(dS0, state_bytes, dST, state_bytes))
        return fail(GDN2_ERR_INVALID_ARG, "%s", "dS0 overlaps dST");
    if (T == 0) {          // no tokens: dS0 = dST
        if (!dS0) return GDN2_OK;
        cudaError_t err = dST ? cudaMemcpyAsync(dS0, dST, state_bytes, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(dS0, 0, state_bytes, s);
        return cuda_status(err, "T = 0 gradient copy");
    }
    const size_t es = dt == GDN2_BF16 ? 2 : 4;
    const size_t tok = (size_t)B * T * H;
    const void *ins[9] = {q, k, v, alpha, b, w, dO, S0, dST};
    const char *in_names[9] = {"q", "k", "v", "alpha", "b", "w", "dO", "S0", "dST"};
    const size_t in_bytes[9] = {tok * d_k * es, tok * d_k * es, tok * d_v * es, tok * d_k * 4, tok * d_k * 4,
                                tok * d_v * 4,  tok * d_v * es, state_bytes,    state_bytes};
    for (int i = 0; i < 7; ++i)
        if ((st = check_ptr(ins[i], in_names[i])) != GDN2_OK) return st;
    if (S0 && (st = check_ptr(S0, "S0")) != GDN2_OK) return st;
    void *outs[8] = {dq, dk, dv, dalpha, db, dw, dS0, workspace};
    const char *out_names[8] = {"dq", "dk", "dv", "dalpha", "db", "dw", "dS0", "workspace"};
    const size_t need = gdn2::chunk_bwd_workspace_floats(B, T, H, d_k, d_v) * sizeof(float);
    const size_t out_bytes[8] = {tok * d_k * es, tok * d_k * es, tok * d_v * es, tok * d_k * 4,
                                 tok * d_k * 4,  tok * d_v * 4,  state_bytes,    need};
    for (int i = 0; i < 8; ++i)
        if (i != 6 && (st = check_ptr(outs[i], out_names[i])) != GDN2_OK) return st;
    if (workspace_bytes < need) return fail(GDN2_ERR_INVALID_ARG, "%s", "workspace smaller than gdn2_chunk_bwd_workspace_size");
    for (int o = 0; o < 8; ++o) {
        for (int i = 0; i < 9; ++i)
            if (overlaps(outs[o], out_bytes[o], ins[i], in_bytes[i]))
                return fail(GDN2_ERR_INVALID_ARG, "%s overlaps an input", out_names[o]);
        for (int o2 = o + 1; o2 < 8; ++o2)
            if (overlaps(outs[o], out_bytes[o], outs[o2], out_bytes[o2]))
                return fail(GDN2_ERR_INVALID_ARG, "%s overlaps another output or the workspace", out_names[o]);
    }
    cudaError_t err = gdn2::launch_chunk_bwd(q, k, v, alpha, b, w, S0, dO, dST, dq, dk, dv, dalpha, db, dw, dS0,
                                             static_cast<float *>(workspace), B, T, H, d_k, d_v, dt, s);
    return cuda_status(err, "gdn2_chunk_bwd launch");
}

gdn2_status gdn2_chunk_fwd_logits(const void *xq, const void *xk, const void *xv, const void *xa, const void *xb,
                                  const void *xw, const float *S0, void *o, float *S_T, int B, int T, int H,
                                  int d_k, int d_v, void *stream) {
    g_last_error[0] = 0;
    gdn2_status st = check_common(B, H, d_k, d_v, GDN2_BF16);
    if (st != GDN2_OK) return st;
    if (d_k != 128 || d_v != 128)
        return fail(GDN2_ERR_UNSUPPORTED, "%s", "gdn2_chunk_fwd_logits: d_k = d_v = 128 only");
    if (T < 0) return fail(GDN2_ERR_INVALID_ARG, "%s", "negative T");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (B == 0 || H == 0) return GDN2_OK;
    const size_t state_bytes = (size_t)B * H * d_k * d_v * sizeof(float);
    if (S0 && (st = check_ptr(S0, "S0")) != GDN2_OK) return st;
    if (S_T && (st = check_ptr(S_T, "S_T")) != GDN2_OK) return st;
    if (S0 && S_T && S0 != S_T && overlaps(S0, state_bytes, S_T, state_bytes))
        return fail(GDN2_ERR_INVALID_ARG, "%s", "S_T partially overlaps S0 (only exact aliasing is allowed)");
    if (T == 0) {
        if (!S_T || S_T == S0) return GDN2_OK;
        cudaError_t err = S0 ? cudaMemcpyAsync(S_T, S0, state_bytes, cudaMemcpyDeviceToDevice, s)
                             : cudaMemsetAsync(S_T, 0, state_bytes, s);
        return cuda_status(err, "T = 0 state copy");
    }
    const void *ins[6] = {xq, xk, xv, xa, xb, xw};
    const char *names[6] = {"xq", "xk", "xv", "xa", "xb", "xw"};
    const size_t row_bytes = (size_t)B * T * H * 128 * 2;      // every logit tensor is [B][T][H][128] BF16
    for (int i = 0; i < 6; ++i)
        if ((st = check_ptr(ins[i], names[i])) != GDN2_OK) return st;
    if ((st = check_ptr(o, "o")) != GDN2_OK) return st;
    for (int i = 0; i < 6; ++i) {
        if (overlaps(o, row_bytes, ins[i], row_bytes)) return fail(GDN2_ERR_INVALID_ARG, "o overlaps %s", names[i]);
        if (S_T && overlaps(S_T, state_bytes, ins[i], row_bytes))
            return fail(GDN2_ERR_INVALID_ARG, "S_T overlaps %s", names[i]);
    }
    if (overlaps(o, row_bytes, S0, state_bytes) || overlaps(o, row_bytes, S_T, state_bytes))
        return fail(GDN2_ERR_INVALID_ARG, "%s", "o overlaps a state buffer");
    cudaError_t err = gdn2::launch_chunk_tc(xq, xk, xv, xa, xb, xw, S0, o, S_T, B, T, H, nullptr, true, s);
    return cuda_status(err, "gdn2_chunk_fwd_logits launch");
}

gdn2_status gdn2_output_gate(const void *o, const void *g, const float *weight, float eps, void *y, int B, int T,
                             int H, int d_v, gdn2_dtype dt, void *stream) {
    g_last_error[0] = 0;
    if (B < 0 || T < 0 || H < 0) return fail(GDN2_ERR_INVALID_ARG, "%s", "negative size");
    if (dt != GDN2_BF16 && dt != GDN2_FP32) return fail(GDN2_ERR_UNSUPPORTED, "%s", "unknown dtype");
    if (d_v != 64 && d_v != 128) return fail(GDN2_ERR_UNSUPPORTED, "%s", "d_v must be 64 or 128");
    if (!(eps >= 0.f) || eps > 3.0e38f) return fail(GDN2_ERR_INVALID_ARG, "%s", "eps must be finite and >= 0");
    const long long rows = (long long)B * T * H;
    if (rows == 0) return GDN2_OK;
    gdn2_status st;
    if ((st = check_ptr(o, "o")) != GDN2_OK || (st = check_ptr(g, "g")) != GDN2_OK ||
        (st = check_ptr(weight, "weight")) != GDN2_OK || (st = check_ptr(y, "y")) != GDN2_OK)
        return st;
    const size_t bytes = (size_t)rows * d_v * (dt == GDN2_BF16 ? 2 : 4);
    if (y != o && overlaps(y, bytes, o, bytes))
        return fail(GDN2_ERR_INVALID_ARG, "%s", "y partially overlaps o (only exact aliasing is allowed)");
    if (overlaps(y, bytes, g, bytes)) return fail(GDN2_ERR_INVALID_ARG, "%s", "y overlaps g");
    if (overlaps(y, bytes, weight, (size_t)d_v * sizeof(float)))
        return fail(GDN2_ERR_INVALID_ARG, "%s", "y overlaps weight");
    return cuda_status(gdn2::launch_output_gate(o, g, weight, eps, y, rows, d_v, dt, static_cast<cudaStream_t>(stream)),
                       "gdn2_output_gate launch");
}

gdn2_status gdn2_recurrent_step(const void *q, const void *k, const void *v, const float *alpha,
                                const float *b, const float *w, float *S, void *o, int B, int H, int d_k,
                                int d_v, gdn2_dtype dt, void *stream) {
    g_last_error[0] = 0;
    gdn2_status st = check_common(B, H, d_k, d_v, dt);
    if (st != GDN2_OK) return st;
    if (B == 0 || H == 0) return GDN2_OK;
    const void *ins[6] = {q, k, v, alpha, b, w};
    const char *names[6] = {"q", "k", "v", "alpha", "b", "w"};
    for (int i = 0; i < 6; ++i)
        if ((st = check_ptr(ins[i], names[i])) != GDN2_OK) return st;
    if ((st = check_ptr(S, "S")) != GDN2_OK) return st;
    if ((st = check_ptr(o, "o")) != GDN2_OK) return st;
    const size_t es = dt == GDN2_BF16 ? 2 : 4;
    const size_t bh = (size_t)B * H;
    const size_t state_bytes = bh * d_k * d_v * sizeof(float);
    const size_t in_bytes[6] = {bh * d_k * es, bh * d_k * es, bh * d_v * es, bh * d_k * 4, bh * d_k * 4, bh * d_v * 4};
    const size_t o_bytes = bh * d_v * es;
    for (int i = 0; i < 6; ++i) {
        if (overlaps(o, o_bytes, ins[i], in_bytes[i])) return fail(GDN2_ERR_INVALID_ARG, "o overlaps %s", names[i]);
        if (overlaps(S, state_bytes, ins[i], in_bytes[i])) return fail(GDN2_ERR_INVALID_ARG, "S overlaps %s", names[i]);
    }
    if (overlaps(o, o_bytes, S, state_bytes)) return fail(GDN2_ERR_INVALID_ARG, "%s", "o overlaps S");
    cudaError_t err = gdn2::launch_recurrent_step(q, k, v, alpha, b, w, S, o, B, H, d_k, d_v, dt,
                                                  static_cast<cudaStream_t>(stream));
    return cuda_status(err, "gdn2_recurrent_step launch");
}

}  // extern "C"
