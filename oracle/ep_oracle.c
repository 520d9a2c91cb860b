/*
 * ep_oracle.c -- CPU oracle for MoE expert-parallel dispatch and combine.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the plain, slow statement of what
 * the dispatch and combine calls compute. It exists so that tests, the smoke
 * check and the CPU baseline of the bench can check the CUDA path against it.
 * Nothing in the product links or calls it, and it shares no header, helper,
 * table or constant with the CUDA path.
 *
 * It is built twice: single-threaded, and with OpenMP (-fopenmp), where the
 * destinations of dispatch and the tokens of combine are shared out over the
 * host's cores. Every output element is computed by the same steps in the
 * same order in both builds, so their results are identical; the OpenMP build
 * only times the same definition on all cores.
 *
 * Sources (mori pages):
 *   - "MORI JIT v2" design page, §3.2 (EpCfg: worldSize, hiddenDim,
 *     maxTokPerRank, numExpertPerRank, numExpertPerToken, maxRecv with
 *     0 meaning worldSize*maxTokPerRank and serving as the stride of the flat
 *     receive index, dtype, useWeights), §3.5 (validity rules), §3.7 (dispatch
 *     moves bytes only; combine reduces), §8 (destPe = expert / numExpertPerRank).
 *   - mori PR #599 "Perf/ep disp 1250 ship", the per-optimisation list:
 *     dedup of (token, destPe), the per-destination histogram, the
 *     three-field per-token meta record, the receive count that is stored
 *     rather than accumulated.
 *
 * Readings where the pages leave a step open (each one is also listed in the
 * design notes of the repository):
 *   - Slots of one destination are ordered by (source rank, source token)
 *     ascending. The pages reserve slots with an atomic fetch_add, whose order
 *     is not defined.
 *   - A token's set of destinations P(r,t) is the set of destPe over its valid
 *     topk entries; an entry < 0 is masked; an entry >= E is a contract
 *     violation: it is reported in the status word and treated as masked.
 *   - Per-destination weight w(r,t,pe) = fold over topk position j ascending
 *     of s = s + w_j (float32, s0 = +0.0f) over the entries that map to pe;
 *     1.0f when useWeights is 0.
 *   - Meta record per (pe, slot), array of structs with 3 + k int32 fields:
 *     source rank, source token, weight sum (float32 bits), then for every topk
 *     position j the local expert id (expert - pe*numExpertPerRank) when entry
 *     j maps to pe, else -1.
 *   - Combine: out[r][t] = bf16_rne( fold over pe in P(r,t) ascending of
 *     acc = fmaf(w(r,t,pe), y[pe][slot], acc) ), acc0 = +0.0f; a token with an
 *     empty P gets a zero row.
 *   - Receive rows and meta past recv_count[pe] are not written.
 *   - Payload dtype (design page §3.7: the dtype is a property of the
 *     transport; dispatch never computes on elements): bf16 2 bytes, fp32 4,
 *     fp8 1, fp4x2 1 byte per element, where an fp4x2 element is a packed pair
 *     of e2m1 values and hiddenDim counts bytes. Dispatch copies rows of
 *     hiddenDim * size bytes. The combine leg reduces, so it takes no byte
 *     type: it is float32 (in and out, no final rounding) for an fp32 plan and
 *     bfloat16 otherwise, with hiddenDim elements, or 2 * hiddenDim for fp4x2
 *     (the unpacked element count) -- the pages pair fp8/fp4 dispatch with a
 *     bf16 combine.
 *
 * Floating point: the pages fix float32 accumulation with bfloat16 output, so
 * the oracle computes in float32 with one fused multiply-add per term (C99
 * fmaf, correctly rounded) and converts with round-to-nearest-even. Build with
 * -ffp-contract=off so that the compiler fuses nothing else.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t worldSize;
    int32_t hiddenDim;
    int32_t maxTokPerRank;
    int32_t numExpertPerRank;
    int32_t numExpertPerToken;
    int32_t maxRecv;
    int32_t dtype;
    int32_t useWeights;
} OracleCfg;

enum {
    ORACLE_OK = 0,
    ORACLE_ERR_ARG = -1,
    ORACLE_ERR_NOMEM = -2,
    ORACLE_STATUS_EXPERT_RANGE = 1, /* positive: an id >= E was seen (masked) */
};

/* bfloat16 <-> float32, from the formats: bf16 is the top half of a float32. */
static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a float32 to bfloat16, nearest with ties to even. A NaN keeps its sign
 * and is forced quiet. */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lower = u & 0xffffu;
    uint32_t upper = u >> 16;
    /* above half: round up; exactly half: round up only when upper is odd */
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;
    return (uint16_t)upper;
}

enum { DT_BF16 = 0, DT_FP32 = 1, DT_FP8 = 2, DT_FP4X2 = 3 };

static int cfg_ok(const OracleCfg *c)
{
    if (!c) return 0;
    if (c->worldSize <= 0 || c->hiddenDim <= 0 || c->maxTokPerRank <= 0) return 0;
    if (c->numExpertPerRank <= 0 || c->numExpertPerToken <= 0) return 0;
    if (c->dtype < DT_BF16 || c->dtype > DT_FP4X2) return 0;
    return 1;
}

/* Bytes of one dispatched element. */
static int64_t payload_size(const OracleCfg *c)
{
    return c->dtype == DT_FP32 ? 4 : c->dtype == DT_BF16 ? 2 : 1;
}

/* Elements of one combine row. */
static int64_t combine_hidden(const OracleCfg *c)
{
    return c->dtype == DT_FP4X2 ? 2 * (int64_t)c->hiddenDim : c->hiddenDim;
}

static int64_t recv_cap(const OracleCfg *c)
{
    return c->maxRecv == 0 ? (int64_t)c->worldSize * c->maxTokPerRank : c->maxRecv;
}

int oracle_recv_capacity(const OracleCfg *c)
{
    return cfg_ok(c) ? (int)recv_cap(c) : ORACLE_ERR_ARG;
}

/*
 * Dispatch. Shapes (all row-major, C order); a row is h * payload_size bytes:
 *   x          bytes  [W][T][row]        the payload, moved bit for bit
 *   topk_idx   int32  [W][T][k]
 *   topk_w     float  [W][T][k]          may be NULL when useWeights == 0
 *   recv_x     bytes  [W][R][row]        R = maxRecv (or W*T)
 *   recv_meta  int32  [W][R][3+k]
 *   recv_count int32  [W]
 *   slotmap    int32  [W][T][W]          slot of (r,t) at pe, or -1
 *   wsum       float  [W][T][W]          w(r,t,pe), 0 where absent
 * Returns 0, ORACLE_STATUS_EXPERT_RANGE when an id >= E was masked, or a
 * negative error.
 */
static int dispatch_impl(const OracleCfg *c, const uint8_t *x, const int32_t *topk_idx,
                         const float *topk_w, const uint32_t *scales, int64_t scale_words,
                         uint8_t *recv_x, int32_t *recv_meta, uint32_t *recv_scales,
                         int32_t *recv_count, int32_t *slotmap, float *wsum);

int oracle_dispatch(const OracleCfg *c, const uint8_t *x, const int32_t *topk_idx,
                    const float *topk_w, uint8_t *recv_x, int32_t *recv_meta,
                    int32_t *recv_count, int32_t *slotmap, float *wsum)
{
    return dispatch_impl(c, x, topk_idx, topk_w, NULL, 0, recv_x, recv_meta, NULL, recv_count,
                         slotmap, wsum);
}

/*
 * Dispatch with a per-token scale row (mori PR #599, its follow-up commits: the
 * scale transport -- a fourth per-token field and the scale row carried with
 * the payload). scales is [W][T][scale_words] 4-byte words; every received row
 * gets its token's scale row at recv_scales [W][R][scale_words], bit for bit,
 * like the payload. Rows past recv_count are not written.
 */
int oracle_dispatch_scaled(const OracleCfg *c, const uint8_t *x, const int32_t *topk_idx,
                           const float *topk_w, const uint32_t *scales, int64_t scale_words,
                           uint8_t *recv_x, int32_t *recv_meta, uint32_t *recv_scales,
                           int32_t *recv_count, int32_t *slotmap, float *wsum)
{
    if (scale_words <= 0 || !scales || !recv_scales) return ORACLE_ERR_ARG;
    return dispatch_impl(c, x, topk_idx, topk_w, scales, scale_words, recv_x, recv_meta,
                         recv_scales, recv_count, slotmap, wsum);
}

static int dispatch_impl(const OracleCfg *c, const uint8_t *x, const int32_t *topk_idx,
                         const float *topk_w, const uint32_t *scales, int64_t scale_words,
                         uint8_t *recv_x, int32_t *recv_meta, uint32_t *recv_scales,
                         int32_t *recv_count, int32_t *slotmap, float *wsum)
{
    if (!cfg_ok(c) || !x || !topk_idx || !recv_x || !recv_meta || !recv_count ||
        !slotmap || !wsum)
        return ORACLE_ERR_ARG;
    if (c->useWeights && !topk_w) return ORACLE_ERR_ARG;

    const int64_t W = c->worldSize, T = c->maxTokPerRank;
    const int64_t row = (int64_t)c->hiddenDim * payload_size(c);
    const int64_t nEpr = c->numExpertPerRank, k = c->numExpertPerToken;
    const int64_t E = W * nEpr, R = recv_cap(c), M = 3 + k;
    int status = ORACLE_OK;
    int overflow = 0;

    /* Every destination hands out its slots in (source rank, source token)
     * ascending order, independently of the other destinations: destination pe
     * counts n from 0 over the tokens that reach it. Built with OpenMP, the
     * destinations run side by side; each writes only its own slots, receive
     * rows, meta records and slot-map column, by the same steps. */
#pragma omp parallel for schedule(dynamic, 1) reduction(| : status, overflow)
    for (int64_t pe = 0; pe < W; ++pe) {
        int64_t n = 0;
        for (int64_t r = 0; r < W; ++r) {
            for (int64_t t = 0; t < T; ++t) {
                const int64_t g = r * T + t;
                const int32_t *ids = topk_idx + g * k;
                int hit = 0;
                float s = 0.0f;
                for (int64_t j = 0; j < k; ++j) {
                    int32_t e = ids[j];
                    if (e < 0) continue;
                    if (e >= E) { status |= ORACLE_STATUS_EXPERT_RANGE; continue; }
                    if (e / nEpr != pe) continue;
                    hit = 1;
                    if (c->useWeights) s = s + topk_w[g * k + j];
                }
                if (!c->useWeights) s = 1.0f;
                if (!hit) {
                    slotmap[g * W + pe] = -1;
                    wsum[g * W + pe] = 0.0f;
                    continue;
                }
                if (n >= R) { overflow = 1; continue; }
                const int64_t slot = n++;
                memcpy(recv_x + (pe * R + slot) * row, x + g * row, (size_t)row);
                if (scales)
                    memcpy(recv_scales + (pe * R + slot) * scale_words, scales + g * scale_words,
                           (size_t)scale_words * sizeof(uint32_t));
                int32_t *meta = recv_meta + (pe * R + slot) * M;
                meta[0] = (int32_t)r;
                meta[1] = (int32_t)t;
                memcpy(&meta[2], &s, sizeof s);
                for (int64_t j = 0; j < k; ++j) {
                    int32_t e = ids[j];
                    meta[3 + j] = (e >= 0 && e < E && e / nEpr == pe) ? (int32_t)(e - pe * nEpr) : -1;
                }
                slotmap[g * W + pe] = (int32_t)slot;
                wsum[g * W + pe] = s;
            }
        }
        recv_count[pe] = (int32_t)n;
    }
    if (overflow) return ORACLE_ERR_ARG; /* more rows than maxRecv at some destination */
    return status;
}

/*
 * Combine. y is [W][R][hc] and out [W][T][hc], hc = combine_hidden: float32
 * for an fp32 plan, bf16 bits (uint16) otherwise; slotmap and wsum are what
 * oracle_dispatch wrote.
 */
int oracle_combine(const OracleCfg *c, const void *y_, const int32_t *slotmap,
                   const float *wsum, void *out_)
{
    if (!cfg_ok(c) || !y_ || !slotmap || !wsum || !out_) return ORACLE_ERR_ARG;
    const int64_t W = c->worldSize, T = c->maxTokPerRank, h = combine_hidden(c);
    const int64_t R = recv_cap(c);
    const int fp32 = c->dtype == DT_FP32;
    const uint16_t *y = (const uint16_t *)y_;
    const float *yf = (const float *)y_;
    uint16_t *out = (uint16_t *)out_;
    float *outf = (float *)out_;
    int nomem = 0;

    /* Built with OpenMP, the tokens are spread over the host's cores; each
     * output row is the same fold in the same order either way. */
#pragma omp parallel
    {
        float *acc = (float *)malloc((size_t)h * sizeof *acc);
#pragma omp for schedule(static) reduction(| : nomem)
        for (int64_t g = 0; g < W * T; ++g) {
            if (!acc) { nomem = 1; continue; }
            for (int64_t i = 0; i < h; ++i) acc[i] = 0.0f;
            for (int64_t pe = 0; pe < W; ++pe) {
                const int32_t slot = slotmap[g * W + pe];
                if (slot < 0) continue;
                const float w = wsum[g * W + pe];
                if (fp32) {
                    const float *rowf = yf + (pe * R + slot) * h;
                    for (int64_t i = 0; i < h; ++i) acc[i] = fmaf(w, rowf[i], acc[i]);
                } else {
                    const uint16_t *row = y + (pe * R + slot) * h;
                    for (int64_t i = 0; i < h; ++i) acc[i] = fmaf(w, bf16_to_f32(row[i]), acc[i]);
                }
            }
            if (fp32)
                for (int64_t i = 0; i < h; ++i) outf[g * h + i] = acc[i];
            else
                for (int64_t i = 0; i < h; ++i) out[g * h + i] = f32_to_bf16_rne(acc[i]);
        }
        free(acc);
    }
    return nomem ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* Threads a call may use: the OpenMP build's team size, 1 otherwise. */
int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* The two format conversions, exported so that tests can pin them against an
 * independent implementation. */
void oracle_f32_to_bf16(const float *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}

void oracle_bf16_to_f32(const uint16_t *in, float *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_to_f32(in[i]);
}
