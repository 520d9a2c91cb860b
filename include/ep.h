/*
 * ep.h -- C ABI of the B200 (sm_100a) MoE expert-parallel dispatch / combine
 * library (libep_b200.so).
 *
 * What the calls compute (mori pages: the "MORI JIT v2" design page and mori
 * PR #599 "Perf/ep disp 1250 ship"):
 *
 *   The W expert-parallel ranks are virtual: every rank's send rows, receive
 *   rows and metadata are regions of one GPU's memory.
 *
 *   dispatch  For every source rank r and token t, every valid topk entry j
 *             (expert id e >= 0) maps to the destination rank
 *             destPe = e / numExpertPerRank (design page §8). The token is sent
 *             once to each distinct destination (dedup of (token, destPe),
 *             PR #599 "ballot dedup"). Destination pe numbers its rows by
 *             (source rank, source token) ascending; row `slot` of pe lives at
 *             flat index pe*maxRecv + slot (design page §3.2: maxRecv is the
 *             stride of the flat receive index). Each row carries a meta record
 *             (PR #599: three per-token fields, here followed by the local
 *             expert ids). The receive count of each destination is stored,
 *             not accumulated (PR #599, follow-up commits: the count is a store).
 *   combine   out[r][t] = bf16_rne( fold over pe in P(r,t) ascending of
 *             acc = fma(w(r,t,pe), float(y[pe][slot]), acc) ), acc0 = +0.0f,
 *             with w(r,t,pe) = float32 sum, in topk order, of the token's topk
 *             weights whose expert lives on pe (1.0f when useWeights == 0);
 *             tokens routed nowhere get a zero row (design page §3.7: combine
 *             reduces, dispatch only moves bytes).
 *
 * Conventions (design page §6): every entry point is noexcept; an error is a
 * NULL or negative return, with a human-readable reason in ep_last_error().
 * Only pointers and scalars cross the boundary.
 *
 * Readings where the pages leave a step open: slot order (the pages reserve
 * slots with an atomic fetch_add, whose order is unspecified; here it is
 * (source rank, source token) ascending, so results are deterministic); an
 * expert id < 0 is a masked entry, so a token whose ids are all < 0 is absent;
 * an expert id >= W*numExpertPerRank is a contract violation, reported through
 * the device error word and treated as masked.
 */
#ifndef EP_B200_H
#define EP_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Payload dtype tags, numbered as the design page's EpDType (§3.7). The dtype is
 * a property of the transport: dispatch moves hiddenDim elements per row bit for
 * bit and never computes on them (bf16 2 bytes, fp32 4, fp8 1, fp4x2 1 byte
 * holding a packed pair of e2m1 values, so hiddenDim counts bytes). The combine
 * leg reduces, so it takes no byte type: it is float32 (in and out, no final
 * rounding) for an EP_FP32 plan and bfloat16 otherwise, with hiddenDim
 * elements per row, or 2 * hiddenDim for EP_FP4X2 (the unpacked count) -- the
 * pages pair fp8/fp4 dispatch with a bf16 combine. */
typedef enum EpDType { EP_BF16 = 0, EP_FP32 = 1, EP_FP8 = 2, EP_FP4X2 = 3 } EpDType;

/* The semantic fields of the design page's EpCfg (§3.2). Launch geometry is
 * not part of it: the library picks it from the device. */
typedef struct EpCfg {
    int32_t worldSize;         /* W: virtual EP ranks, 1..32 */
    int32_t hiddenDim;         /* h: payload elements per token row; its bytes must be a multiple of 16 */
    int32_t maxTokPerRank;     /* T: token rows per source rank, >= 1 */
    int32_t numExpertPerRank;  /* experts on each rank, >= 1; E = W*numExpertPerRank */
    int32_t numExpertPerToken; /* k (topk), 1..32 */
    int32_t maxRecv;           /* receive rows per destination; 0 means W*T; must be >= W*T */
    int32_t dtype;             /* EpDType of the dispatch payload (see above) */
    int32_t useWeights;        /* 1: combine weights by the topk weights; 0: weight 1 */
} EpCfg;

/* What a plan resolved. Sizes are in bytes. */
typedef struct EpPlanInfo {
    int32_t maxRecv;          /* resolved receive capacity per destination */
    int32_t metaFields;       /* int32 fields per meta record: 3 + k */
    int64_t rowBytes;         /* bytes of a dispatched row: h * element size */
    int64_t tokenBytes;       /* bytes of x: W*T*rowBytes */
    int64_t recvXBytes;       /* bytes of recv_x: W*maxRecv*rowBytes */
    int64_t recvMetaBytes;    /* W*maxRecv*metaFields*4 */
    int64_t scratchBytes;     /* device scratch the plan owns */
    int32_t countTile;        /* tokens per routing tile */
    int32_t numTiles;         /* routing tiles: ceil(W*T / countTile) */
    int32_t scatterBlocks;    /* grid of the row-scatter kernel */
    int32_t scatterWarps;     /* copy engines (warps) per scatter block */
    int32_t scatterStages;    /* shared-memory stages per copy engine */
    int32_t scatterChunkBytes;/* bytes per staged copy (a row, or a piece of one) */
    int32_t combineBlocks;    /* grid of the combine kernel */
    int32_t combineWarps;     /* warps per combine block */
    int32_t device;           /* CUDA device the plan lives on (-1 from ep_plan_query) */
    int32_t numSMs;           /* SMs of that device (0 from ep_plan_query) */
    int32_t scatterMode;      /* 0: TMA bulk copies staged in shared memory (the only mode) */
    int32_t scatterPend;      /* bulk-store groups left draining when a stage refills (1) */
    int32_t combineDtype;     /* EP_FP32 for an fp32 plan, else EP_BF16 */
    int32_t combineHidden;    /* elements of a y / out row: h, or 2*h for EP_FP4X2 */
    int64_t combineRowBytes;  /* bytes of a y / out row */
    int64_t yBytes;           /* bytes of y: W*maxRecv*combineRowBytes */
    int64_t outBytes;         /* bytes of out: W*T*combineRowBytes */
    int32_t dispatchFused;    /* 1: dispatch is one launch (EP_DISPATCH_FUSED=1, where every
                                 block owns at most 64 tokens): block b routes its own
                                 contiguous share of the W*T tokens (scatterBlocks blocks),
                                 publishes its per-destination totals, adds up the earlier
                                 blocks' totals (decoupled look-back, a bounded wait) and
                                 copies its own tokens; 0: two launches (route_count,
                                 scatter_rows). Results are identical either way. The
                                 one-launch form suits full, small batches (up to ~20
                                 tokens a block): where only the first tokens of each rank
                                 are live, a few blocks do all the copies. */
    int32_t combineLoadBytes; /* 32: the combine reads y in 32-byte loads (outBytes of at
                                 least 192 MiB, combine rows a multiple of 32 bytes; a call
                                 whose y is not 32-byte aligned takes 16-byte loads); 16
                                 otherwise. Results are identical either way. */
} EpPlanInfo;

typedef struct EpPlan EpPlan;

/* Return codes (negative) of the host entry points. */
enum {
    EP_OK = 0,
    EP_ERR_INVALID = -1,     /* bad argument or configuration */
    EP_ERR_UNSUPPORTED = -2, /* valid for the pages, not built here */
    EP_ERR_NOMEM = -3,       /* device allocation failed */
    EP_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed */
    EP_ERR_STATE = -5,       /* combine before any dispatch on this plan */
    EP_ERR_ALIGN = -6,       /* a buffer is not aligned as documented */
    EP_ERR_DEVICE = -7       /* the current device is not the plan's device */
};

/* Bits of the device error word (ep_plan_check_error). Kernels never trap:
 * they record the problem here and keep going or return. */
enum {
    EP_DEVERR_EXPERT_RANGE = 1, /* an expert id >= E was seen; it was treated as masked */
    EP_DEVERR_TIMEOUT = 2,      /* a bounded wait gave up: on a copy's shared-memory barrier,
                                   on another block's published totals (dispatchFused), or on
                                   another rank's barrier flag (ep_comm.h) */
    EP_DEVERR_CAPACITY = 4,     /* a destination received more than maxRecv rows */
    EP_DEVERR_BOUNDS = 8        /* bounds-checking build only (libep_b200_debug.so): an access
                                   fell outside its buffer; it was skipped */
};

/* Validate a configuration on the host (no CUDA call). Returns EP_OK, or
 * EP_ERR_INVALID / EP_ERR_UNSUPPORTED with the reason in ep_last_error().
 * Rules (design page §3.5, EpCfgIsValid): the row bytes must be a multiple of
 * 16; topk and worldSize must fit one 32-lane warp; the receive capacity must
 * cover the worst case (maxRecv >= W*T); dtype one of EpDType (§3.7). */
int ep_cfg_check(const EpCfg* cfg);

/* Host-only sizing: fill *info for cfg as a plan on a generic device would
 * resolve it (device = -1, numSMs = 0, geometry from a 148-SM B200 without
 * the geometry overrides; EP_DISPATCH_FUSED and EP_COMBINE_WIDE are
 * honoured). Lets a
 * caller size recv_x / recv_meta before creating a plan. Returns EP_OK or a
 * negative code. */
int ep_plan_query(const EpCfg* cfg, EpPlanInfo* info);

/* Create a plan on the current CUDA device: validates cfg, picks the launch
 * geometry, allocates and zeroes the plan's device scratch (routing table
 * [W*T][W] of (slot, weight) pairs, per-tile counts and offsets, a tile
 * ticket, the error word). Returns NULL on failure (ep_last_error() says why).
 * Environment overrides, read here only (for geometry sweeps):
 * EP_SCATTER_BLOCKS, EP_SCATTER_WARPS, EP_SCATTER_STAGES, EP_SCATTER_CHUNK, EP_COMBINE_BLOCKS,
 * EP_COMBINE_WARPS, EP_DISPATCH_FUSED (1: the one-launch dispatch of
 * dispatchFused, where every block owns at most 64 tokens; off by default),
 * EP_SCATTER_FANOUT_SWITCH (100 x
 * the mean fan-out above which one copy engine per block sits out; 375 by
 * default, 0 never), EP_SCATTER_SCAN ("route": route_count's last block scans
 * the tile counts even when the scatter could), EP_DISPATCH_DENSE (1 / 0: the
 * large-batch form of the split dispatch for every plan / for none; by default
 * plans of more than 16384 tokens, W*T, take it), EP_COMBINE_WIDE (1 / 0:
 * 32-byte combine loads for every plan whose combine rows are a multiple of
 * 32 bytes / for none; by default plans whose outBytes is at least 192 MiB). Test hooks:
 * EP_TEST_UNREACHABLE_BARRIER=1 makes the one-launch dispatch's wait for the
 * earlier blocks' totals unreachable, so that the bounded wait runs out: every
 * block but the first (which waits on nothing and copies its own tokens)
 * reports EP_DEVERR_TIMEOUT, copies nothing and returns about one second
 * later, and the context stays usable; EP_TEST_BOUNDS_ROWS=n makes the bounds-checking
 * build (libep_b200_debug.so) check the receive buffers against n rows per
 * destination instead of maxRecv. */
EpPlan* ep_plan_create(const EpCfg* cfg);

/* Free the plan and its scratch. NULL is a no-op. The caller must make sure no
 * dispatch or combine of this plan is still running on the GPU. */
void ep_plan_destroy(EpPlan* plan);

/* Copy the plan's resolved sizes and geometry into *info. */
int ep_plan_info(const EpPlan* plan, EpPlanInfo* info);

/*
 * Dispatch, enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 * stream). No host synchronisation, no allocation: capturable in a CUDA graph.
 * All pointers are device pointers owned by the caller.
 *   x          dtype [W][T][h]            16-byte aligned
 *   topk_idx   int32 [W][T][k]            expert ids; < 0 masked
 *   topk_w     float [W][T][k]            NULL allowed when useWeights == 0
 *   recv_x     dtype [W][maxRecv][h]      16-byte aligned; rows >= recv_count[pe]
 *                                         of destination pe are not written
 *   recv_meta  int32 [W][maxRecv][3+k]    per row: source rank, source token,
 *                                         weight sum (float32 bits), then for
 *                                         each topk position j the local expert
 *                                         id (e - pe*numExpertPerRank) when
 *                                         entry j lives on pe, else -1; records
 *                                         past recv_count are not written
 *   recv_count int32 [W]                  rows received per destination (stored)
 * The routing (slot and weight of every (r,t,pe)) stays in the plan for the
 * next ep_combine. Returns EP_OK or a negative code; kernel-side contract
 * violations go to the device error word.
 */
int ep_dispatch(EpPlan* plan, const void* x, const int32_t* topk_idx, const float* topk_w,
                void* recv_x, int32_t* recv_meta, int32_t* recv_count, void* stream);

/* Largest scale row of ep_dispatch_scaled, in 4-byte words. */
#define EP_MAX_SCALE_WORDS 4096

/*
 * Dispatch with a per-token scale row (mori PR #599, its follow-up commits:
 * the scale transport, a fourth per-token field carried with the payload, as
 * quantized payloads need). Same as ep_dispatch, plus:
 *   scales       [W][T][scaleWords]        4-byte words (e.g. float32 scales),
 *                                          4-byte aligned; moved bit for bit
 *   scaleWords   1..EP_MAX_SCALE_WORDS     (1: one scale per token; h/128 for
 *                                          per-128-element block scales)
 *   recv_scales  [W][maxRecv][scaleWords]  every received row gets its token's
 *                                          scale row; rows past recv_count[pe]
 *                                          are not written
 */
int ep_dispatch_scaled(EpPlan* plan, const void* x, const int32_t* topk_idx, const float* topk_w,
                       const void* scales, int32_t scaleWords, void* recv_x, int32_t* recv_meta,
                       void* recv_scales, int32_t* recv_count, void* stream);

/*
 * Combine, enqueued on `stream`, using the routing of the most recent
 * ep_dispatch of this plan (stream order is the caller's: issue it on the same
 * stream, or order the streams). No host synchronisation, no allocation.
 * A combine may be repeated on the same routing (e.g. for several expert
 * outputs). Calls on one plan share its scratch, so the executions of a
 * plan's dispatches and combines must not overlap on the GPU.
 *   y    [W][maxRecv][hc]  expert outputs in the receive layout, 16-byte
 *                          aligned; only rows < recv_count are read
 *   out  [W][T][hc]        16-byte aligned; every row is written
 * Both are float32 for an EP_FP32 plan and bfloat16 otherwise; hc =
 * combineHidden of ep_plan_info (2*h for EP_FP4X2, else h). A NaN in y gives
 * a NaN out element; its sign and payload bits are not specified.
 * Returns EP_OK, EP_ERR_STATE before any dispatch, or a negative code.
 */
int ep_combine(EpPlan* plan, const void* y, void* out, void* stream);

/* Synchronise the device, return the device error word (a bitmask of
 * EP_DEVERR_*, 0 when clean) and clear it; negative on a CUDA error. Meant for
 * tests and debugging, not for the hot path. */
int ep_plan_check_error(EpPlan* plan);

/* Reason for the last failure on this thread ("" if none). */
const char* ep_last_error(void);

/* Bytes of device scratch that ep_dispatch_noalloc has on each device. */
#define EP_NOALLOC_SCRATCH_BYTES (4 * 1024 * 1024)

/*
 * ep_dispatch_noalloc -- dispatch without a plan and without allocating.
 * The pages have no counterpart of this call; it exists for callers that
 * cannot allocate device memory where they dispatch: a serving loop whose
 * memory pool must not grow, code running inside an allocator or driver
 * callback (allocating there would re-enter the allocator), or an embedder
 * whose runtime owns every device allocation.
 *
 * Same arguments, layouts and results as ep_dispatch (it runs the same
 * kernels), with the configuration passed directly instead of a plan. It
 * calls no cudaMalloc, cudaFree or other allocating routine: its scratch (the
 * routing table, per-tile counts and bases, tile ticket, error word) is one
 * file-scope __device__ array of EP_NOALLOC_SCRATCH_BYTES bytes, which every
 * device that loads the library holds until the process exits.
 *   - Limit: the configuration's scratch (about W*W*maxTokPerRank*8 bytes for
 *     the routing table plus the tile tables) must fit the array; larger
 *     configurations return EP_ERR_INVALID with the sizes in ep_last_error().
 *   - The first call on a device looks up the array's device address and the
 *     device limits (a one-time set-up, with that device current); make that
 *     first call before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; each call clears what must start at zero (tile ticket, error
 *     word) on `stream`. Calls whose executions overlap on the GPU (other
 *     streams, other host threads) race on the array and give wrong results:
 *     serialise them.
 *   - The routing table it leaves is not a plan's, so ep_combine cannot follow
 *     it; device-side contract violations (ids >= E) are masked but not
 *     reported (there is no plan error word to read).
 * Returns EP_OK or a negative code (reason in ep_last_error()).
 */
int ep_dispatch_noalloc(const EpCfg* cfg, const void* x, const int32_t* topk_idx,
                        const float* topk_w, void* recv_x, int32_t* recv_meta,
                        int32_t* recv_count, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_H */
