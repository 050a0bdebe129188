// C ABI entry points (declared in include/reatt.h): argument checks on the
// host, the workspace plan, and the launch sequence of each call.  Nothing
// here allocates device memory; every buffer comes from the caller.
#include <math.h>
#include <string.h>

#include "kernels.h"
#include "reatt.h"

namespace reatt {
namespace {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t up256(size_t x) { return (x + 255) / 256 * 256; }
constexpr int64_t kMaxWindow = int64_t(1) << 24;   // Wmax limit (exact fp32 positions)

int make_geom(const reatt_dims *d, Geom *g)
{
    if (!d || !g) return REATT_EINVAL;
    if (d->B < 1 || d->Hq < 1 || d->Hkv < 1 || d->C < 1 || d->G < 0 || d->L < 0 || d->S < 1 ||
        d->k < 0 || d->T < 0)
        return REATT_EINVAL;
    if (d->Hq % d->Hkv != 0) return REATT_EINVAL;
    if (!(d->rope_base > 0.0) || !isfinite(d->rope_base)) return REATT_EINVAL;
    if (d->dtype != REATT_F32 && d->dtype != REATT_BF16) return REATT_EUNSUPPORTED;
    if (d->d != 64 && d->d != 128) return REATT_EUNSUPPORTED;
    if (d->k > 65536) return REATT_EUNSUPPORTED;
    if (d->T >= (int64_t(1) << 31)) return REATT_EUNSUPPORTED;
    if (d->T_cap != 0 && (d->T_cap < d->T || d->T_cap >= (int64_t(1) << 31))) return REATT_EINVAL;
    const double wmax = double(d->G) + double(d->k) * d->S + d->L + d->C;
    // RoPE angles are formed from the window position in fp32 (rope_cs), which
    // holds every integer position exactly only below 2^24.
    if (wmax > double(kMaxWindow)) return REATT_EUNSUPPORTED;
    // element counts of the largest buffers must fit comfortably in int64
    const double cache = double(d->B) * d->Hkv * double(d->T_cap ? d->T_cap : d->T) * d->d;
    const double win = double(d->B) * d->Hkv * wmax * d->d;
    const double qn = double(d->B) * d->Hq * double(d->C) * d->d;
    if (cache > 4e18 || win > 4e18 || qn > 4e18) return REATT_EUNSUPPORTED;

    g->B = d->B;
    g->Hq = d->Hq;
    g->Hkv = d->Hkv;
    g->g = d->Hq / d->Hkv;
    g->d = d->d;
    g->C = d->C;
    g->G = d->G;
    g->L = d->L;
    g->S = d->S;
    g->k = d->k;
    g->T = d->T;
    g->Ts = d->T_cap ? d->T_cap : d->T;
    g->g_end = d->T < d->G ? d->T : d->G;
    g->loc_begin = (d->T - d->L) > d->G ? (d->T - d->L) : d->G;
    g->n_loc = d->T > g->loc_begin ? d->T - g->loc_begin : 0;
    g->M = d->T - d->G - d->L > 0 ? d->T - d->G - d->L : 0;
    g->NS = (g->M + d->S - 1) / d->S;
    g->Wmax = int64_t(d->G) + int64_t(d->k) * d->S + d->L + d->C;
    g->base = d->rope_base;
    g->dtype = d->dtype;
    for (int i = 0; i < 64; ++i) {
        g->rope_hi[i] = g->rope_lo[i] = 0.f;
        if (i < d->d / 2) {
            const double f = pow(d->rope_base, -2.0 * i / double(d->d)) / M_PI;
            g->rope_hi[i] = float(f);
            g->rope_lo[i] = float(f - double(g->rope_hi[i]));
        }
    }
    return REATT_OK;
}

// Workspace layout: [status header][attention tickets][attention partials]
// [top-k candidates][summed queries (C > 1)][span scores][selection][RoPE table]
// [prefill attention operands].
struct WsPlan {
    size_t ticket, ticket_bytes, topk, qsum, scores, sel, tab, fa, total;
};
WsPlan ws_plan(const Geom &g)
{
    WsPlan p;
    size_t off = kWsHeader;
    size_t tb = 0, mo = 0;
    const size_t attn = attend_ws_bytes(g, &tb, &mo);
    p.ticket = off;
    p.ticket_bytes = tb;
    off = up256(off + attn);
    p.topk = off;
    off = up256(off + topk_ws_bytes(g));
    p.qsum = off;
    off = up256(off + score_spans_ws_bytes(g));
    p.scores = off;
    off = up256(off + size_t(g.B) * g.Hkv * g.NS * sizeof(float));
    p.sel = off;
    off = up256(off + size_t(g.B) * g.Hkv * g.k * sizeof(int32_t));
    p.tab = off;
    off = up256(off + rope_table_bytes(g));
    p.fa = off;
    off = up256(off + prefill_attn_tc_ws_bytes(g));
    p.total = off;
    return p;
}

inline uint8_t *at(void *ws, size_t off) { return static_cast<uint8_t *>(ws) + off; }

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? REATT_OK : REATT_ECUDA; }

}  // namespace

int geom_of(const reatt_dims *d, Geom *g) { return make_geom(d, g); }

}  // namespace reatt

using namespace reatt;

extern "C" {

const char *reatt_status_string(int status)
{
    switch (status) {
    case REATT_OK: return "ok";
    case REATT_EINVAL: return "invalid argument (null/misaligned pointer or bad size)";
    case REATT_EUNSUPPORTED: return "unsupported configuration (head width, dtype or size)";
    case REATT_ECUDA: return "CUDA error while launching";
    case REATT_ETIMEOUT: return "a kernel's bounded wait gave up";
    default: return "unknown status";
    }
}

int reatt_num_spans(const reatt_dims *dims, int64_t *num_spans)
{
    Geom g;
    const int rc = make_geom(dims, &g);
    if (rc) return rc;
    if (!num_spans) return REATT_EINVAL;
    *num_spans = g.NS;
    return REATT_OK;
}

int reatt_window_max(const reatt_dims *dims, int64_t *wmax)
{
    Geom g;
    const int rc = make_geom(dims, &g);
    if (rc) return rc;
    if (!wmax) return REATT_EINVAL;
    *wmax = g.Wmax;
    return REATT_OK;
}

int reatt_workspace_bytes(const reatt_dims *dims, size_t *bytes)
{
    Geom g;
    const int rc = make_geom(dims, &g);
    if (rc) return rc;
    if (!bytes) return REATT_EINVAL;
    *bytes = ws_plan(g).total;
    return REATT_OK;
}

int reatt_workspace_status(void *ws, int *status, reatt_stream stream)
{
    if (!ws || !status || !aligned16(ws)) return REATT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof word, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof word, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return REATT_ECUDA;
    *status = word == 0 ? REATT_OK : int(word);
    return REATT_OK;
}

int reatt_score_spans(const reatt_dims *dims, const void *q, const void *k_cache,
                      float *span_scores, void *ws, reatt_stream stream)
{
    Geom g;
    const int rc = make_geom(dims, &g);
    if (rc) return rc;
    const bool need_k = g.NS > 0;
    if (!q || !ws || (need_k && (!k_cache || !span_scores))) return REATT_EINVAL;
    if (!aligned16(q) || !aligned16(ws) || !aligned16(k_cache) || !aligned16(span_scores))
        return REATT_EINVAL;
    const WsPlan p = ws_plan(g);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    return cuda_status(
        launch_score_spans(g, q, k_cache, span_scores, ws, at(ws, p.qsum), nullptr, st));
}

int reatt_topk(const reatt_dims *dims, const float *span_scores, int32_t *sel, void *ws,
               reatt_stream stream)
{
    Geom g;
    const int rc = make_geom(dims, &g);
    if (rc) return rc;
    if (g.k == 0) return REATT_OK;
    if (!sel || !ws || (g.NS > 0 && !span_scores)) return REATT_EINVAL;
    if (!aligned16(sel) || !aligned16(ws) || !aligned16(span_scores)) return REATT_EINVAL;
    const WsPlan p = ws_plan(g);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    return cuda_status(
        launch_topk(g, span_scores, sel, at(ws, p.topk), nullptr, 0, nullptr, st));
}

int reatt_gather_rope(const reatt_dims *dims, const void *k_cache, const void *v_cache,
                      const void *k_cur, const void *v_cur, const int32_t *sel, float *k_win,
                      float *v_win, int32_t *win_len, reatt_stream stream)
{
    Geom g;
    const int rc = make_geom(dims, &g);
    if (rc) return rc;
    const bool need_cache = g.T > 0;
    if (!k_cur || !v_cur || !k_win || !v_win || !win_len) return REATT_EINVAL;
    if (need_cache && (!k_cache || !v_cache)) return REATT_EINVAL;
    if (g.k > 0 && !sel) return REATT_EINVAL;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_cur) || !aligned16(v_cur) ||
        !aligned16(sel) || !aligned16(k_win) || !aligned16(v_win) || !aligned16(win_len))
        return REATT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    return cuda_status(
        launch_gather_rope(g, k_cache, v_cache, k_cur, v_cur, sel, k_win, v_win, win_len, st));
}

int reatt_attend(const reatt_dims *dims, const void *q, const float *k_win, const float *v_win,
                 const int32_t *win_len, float *out, void *ws, reatt_stream stream)
{
    Geom g;
    const int rc = make_geom(dims, &g);
    if (rc) return rc;
    if (!q || !k_win || !v_win || !win_len || !out || !ws) return REATT_EINVAL;
    if (!aligned16(q) || !aligned16(k_win) || !aligned16(v_win) || !aligned16(win_len) ||
        !aligned16(out) || !aligned16(ws))
        return REATT_EINVAL;
    const WsPlan p = ws_plan(g);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(at(ws, p.ticket), 0, p.ticket_bytes, st);
    if (e != cudaSuccess) return REATT_ECUDA;
    return cuda_status(launch_attend(g, q, k_win, v_win, win_len, nullptr, nullptr, nullptr,
                                     nullptr, nullptr, nullptr, out, at(ws, p.ticket), ws, false,
                                     st));
}

int reatt_step(const reatt_dims *dims, const void *q, const void *k_cache, const void *v_cache,
               const void *k_cur, const void *v_cur, int32_t *sel_out, float *out, void *ws,
               reatt_stream stream)
{
    Geom g;
    const int rc = make_geom(dims, &g);
    if (rc) return rc;
    if (!q || !k_cur || !v_cur || !out || !ws) return REATT_EINVAL;
    if (g.T > 0 && (!k_cache || !v_cache)) return REATT_EINVAL;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_cur) ||
        !aligned16(v_cur) || !aligned16(sel_out) || !aligned16(out) || !aligned16(ws))
        return REATT_EINVAL;
    const WsPlan p = ws_plan(g);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float *scores = reinterpret_cast<float *>(at(ws, p.scores));
    int32_t *sel = sel_out ? sel_out : reinterpret_cast<int32_t *>(at(ws, p.sel));
    float2 *tab = reinterpret_cast<float2 *>(at(ws, p.tab));
    // Decode with a window length that does not depend on the selection: the
    // scan writes the RoPE table and the attention starts on the fixed part
    // of the window while the top-k runs.  Otherwise the top-k launch fills
    // the table.  Either way the top-k launch clears the attention tickets.
    const bool tc_attn = prefill_attn_tc_eligible(g);
    const int64_t w_known = (g.C == 1 && g.NS > 0 && !tc_attn && attn_plan(g).decode)
                                ? decode_window_known(g)
                                : -1;
    bool codes = false;   // the prefill scan may leave order codes for the top-k
    cudaError_t e = launch_score_spans(g, q, k_cache, scores, ws, at(ws, p.qsum),
                                       w_known >= 0 ? tab : nullptr, st, true, &codes);
    if (e != cudaSuccess) return REATT_ECUDA;
    e = launch_topk(g, scores, sel, at(ws, p.topk), reinterpret_cast<uint32_t *>(at(ws, p.ticket)),
                    int(p.ticket_bytes / sizeof(uint32_t)), w_known >= 0 ? nullptr : tab, st,
                    codes);
    if (e != cudaSuccess) return REATT_ECUDA;
    if (tc_attn)   // many query rows: tensor-core attention
        return cuda_status(launch_attend_prefill_tc(g, q, k_cache, v_cache, k_cur, v_cur, sel, tab,
                                                    out, at(ws, p.fa), ws, st));
    return cuda_status(launch_attend(g, q, nullptr, nullptr, nullptr, k_cache, v_cache, k_cur,
                                     v_cur, sel, tab, out, at(ws, p.ticket), ws, true, st,
                                     w_known));
}

int reatt_append_kv(const reatt_dims *dims, void *k_cache, void *v_cache, const void *k_cur,
                    const void *v_cur, reatt_stream stream)
{
    Geom g;
    const int rc = make_geom(dims, &g);
    if (rc) return rc;
    if (g.Ts < g.T + g.C) return REATT_EINVAL;   // the caches have no room for C more rows
    if (!k_cache || !v_cache || !k_cur || !v_cur) return REATT_EINVAL;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_cur) || !aligned16(v_cur))
        return REATT_EINVAL;
    return cuda_status(launch_append(g, k_cache, v_cache, k_cur, v_cur,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
