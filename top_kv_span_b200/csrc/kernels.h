// Host-side launchers of the sm_100a kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "common.cuh"

namespace reatt {

// Launch with programmatic stream serialization: the kernel may begin while
// its predecessor in the stream finishes; it must call pdl_wait() before
// touching anything the predecessor writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args &&...args)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

inline bool geo_is_bf16(const Geom &g) { return g.dtype == REATT_BF16; }

int num_sms();

// Checked geometry of a call (host argument checks of the C ABI).
int geom_of(const reatt_dims *d, Geom *g);

// span scoring: scratch holds the fp32 summed queries when C > 1; rope_tab
// (nullable, decode only) is filled with the step's RoPE table on the side;
// allow_tc = false keeps C > 1 off the tensor-core scan (its tensor maps need
// the cache's own base address).  With codes_left non-null the scores may be
// left as order codes (uint32, see order_code), which *codes_left then says;
// otherwise they are always floats.
size_t score_spans_ws_bytes(const Geom &geo);
cudaError_t launch_score_spans(const Geom &geo, const void *q, const void *kc, float *scores,
                               void *ws, void *scratch, float2 *rope_tab, cudaStream_t st,
                               bool allow_tc = true, bool *codes_left = nullptr);

// prefill span scoring on tcgen05 (bf16, C > 1, S divides 32)
bool prefill_tc_eligible(const Geom &geo);
size_t prefill_tc_ws_bytes(const Geom &geo);
cudaError_t launch_prefill_tc(const Geom &geo, const void *q, const void *kc, float *scores,
                              void *ws, void *scratch, cudaStream_t st, bool *codes_left);

// prefill attention on tcgen05 (bf16, more than 8 query rows per KV head)
bool prefill_attn_tc_eligible(const Geom &geo);
size_t prefill_attn_tc_ws_bytes(const Geom &geo);
cudaError_t launch_attend_prefill_tc(const Geom &geo, const void *q, const void *kc,
                                     const void *vc, const void *kcur, const void *vcur,
                                     const int32_t *sel, const float2 *tab, float *out,
                                     void *scratch, void *ws, cudaStream_t st);

// top-k: scratch holds per-slice candidates when NS is large; zero_words
// (nullable) are cleared by the first CTA (used to reset attention tickets);
// rope_tab (nullable) is filled by spare CTAs of the same launch; with codes
// the scores buffer holds order codes (uint32) instead of floats
size_t topk_ws_bytes(const Geom &geo);
int topk_selecting_ctas(const Geom &geo);   // CTAs of the first top-k launch that select
cudaError_t launch_topk(const Geom &geo, const float *scores, int32_t *sel, void *scratch,
                        uint32_t *zero_words, int nzero, float2 *rope_tab, cudaStream_t st,
                        bool codes = false);
// top-k of candidate lists: per (b, h), ncand order codes and span ids (in
// ascending id order; code 0 = empty) -> the min(k, NS) best ids, ascending
cudaError_t launch_topk_merge(const Geom &geo, const uint32_t *codes, const int32_t *ids,
                              int32_t *sel, int ncand, cudaStream_t st);

// current tokens' K/V rows -> cache rows [T, T + C) (caches of Ts rows per head)
cudaError_t launch_append(const Geom &geo, void *k_cache, void *v_cache, const void *k_cur,
                          const void *v_cur, cudaStream_t st);

cudaError_t launch_gather_rope(const Geom &geo, const void *kc, const void *vc, const void *kcur,
                               const void *vcur, const int32_t *sel, float *kw, float *vw,
                               int32_t *win_len, cudaStream_t st);

// Arguments of the windowed-attention kernels.
struct AttnArgs {
    const void *q;
    const int32_t *sel;       // virtual window
    const int32_t *win_len;   // materialised window
    const float2 *tab;        // virtual window: RoPE cos/sin [Wmax][D/2]
    float *out;
    float *part_acc;          // [BH][nqb][nsplit][QB][D]
    float2 *part_ml;          // [BH][nqb][nsplit][QB] (max, sum)
    uint32_t *ticket;         // [BH][nqb]
    int nqb, nsplit;
    int64_t w_known;          // decode: window length known before the selection, or -1
};

// 2-D tensor map of a row-major bf16 matrix (rows x cols), boxes of
// box_rows x 64 elements, 128-byte swizzle, zero fill out of range.
bool encode_bf16_map(CUtensorMap *mp, const void *base, uint64_t rows, uint64_t cols,
                     uint32_t box_rows);

// Decode attention of the fused step on the tensor cores (bf16, d = 128, at
// most 8 query rows per KV head, every window run a multiple of 8 rows):
// QB = RP query rows per CTA.
bool decode_tc_eligible(const Geom &geo);
cudaError_t launch_attend_decode_tc(const Geom &geo, const AttnArgs &a, int RP, const void *kc,
                                    const void *vc, const void *kcur, const void *vcur, void *ws,
                                    cudaStream_t st);

struct AttnPlan {
    bool decode;   // warp kernel (<= 8 query rows per KV head) or tile kernel
    int QB, nqb, nsplit;
};
// reserved_sms: SMs left to kernels that run beside the attention (the top-k)
AttnPlan attn_plan(const Geom &geo, int reserved_sms = 0);
// bytes of tickets (256-aligned, reported separately) + split-K partials
// (accumulators, then (max, sum) pairs at *ml_off)
size_t attend_ws_bytes(const Geom &geo, size_t *ticket_bytes, size_t *ml_off);
// bytes of the per-step RoPE cos/sin table (Wmax x d/2 float2)
size_t rope_table_bytes(const Geom &geo);
// virt = true: keys/values read from the un-rotated cache through sel and
// rotated with rope_tab; virt = false: from the materialised fp32 window.
cudaError_t launch_attend(const Geom &geo, const void *q, const float *kw, const float *vw,
                          const int32_t *win_len, const void *kc, const void *vc,
                          const void *kcur, const void *vcur, const int32_t *sel,
                          const float2 *rope_tab, float *out, void *scratch, void *ws, bool virt,
                          cudaStream_t st, int64_t w_known = -1);
// Window length of the fused decode step when it does not depend on the
// selection (no ragged last span, or nothing selected), else -1.  With it the
// decode attention takes the fixed part of the window (local rows and the
// current token) before the selection is complete; the RoPE table must then
// be written by the scan.
int64_t decode_window_known(const Geom &geo);

}  // namespace reatt
