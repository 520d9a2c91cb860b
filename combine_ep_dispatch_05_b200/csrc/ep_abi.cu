// ep_abi.cu -- the C ABI of include/ep.h: configuration checks, plans (device
// scratch + launch geometry) and the dispatch / combine entry points.
//
// Conventions follow the "MORI JIT v2" design page §6: every entry point is
// noexcept (no exception crosses extern "C"), errors are NULL / negative
// returns with the reason kept in a thread-local string.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "ep.h"
#include "ep_internal.h"

struct EpPlan {
    EpCfg cfg;
    EpPlanInfo info;
    int device;
    int maxRecv;
    int G;            // W*T
    void* scratch;    // one allocation, carved below
    int2* route;      // [G][W]
    uint32_t* tok_mask;  // [G]
    int32_t* tile_cnt;
    int32_t* tile_base;
    uint32_t* ticket;
    int32_t* work;
    int32_t* ptotal;      // route_count's present-token total (last-block scan)
    int32_t* cwork;
    uint32_t* cdone;
    int32_t* err;
    size_t scatterSmem;
    bool dense;           // large batches: route_count's earlier form, tile bases in global memory
    size_t baseSmem;      // > 0: the scatter scans the tile counts into this much shared memory
    size_t baseOffset;    // its offset in the scatter's shared memory, and the engines'
    size_t engineOffset;
    bool fused;           // the fused dispatch (dispatch_fused): one launch, per-block routing
    size_t fusedSmem;     // its dynamic shared memory: routing area, then the copy engines
    size_t fusedEngineOffset;
    int fusedOwn;         // the most tokens one of its blocks owns
    int fusedBlocks;      // its grid
    unsigned long long* fused_agg;  // its scratch: the blocks' published totals, call epoch, blocks done
    unsigned* fused_epoch;
    unsigned* fused_done;
    unsigned barrierSlack;  // test hook: 1 makes the fused dispatch's look-back unreachable
    int boundsRows;         // bounds-checking build: rows of each destination's buffers it checks against
    int fanoutSwitch;       // x100, see ScatterParams
    bool dispatched;
};

namespace {

thread_local char g_last_error[512] = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(e == cudaErrorMemoryAllocation ? EP_ERR_NOMEM : EP_ERR_CUDA, "%s: %s (%s)", what,
                cudaGetErrorName(e), cudaGetErrorString(e));
}

// An integer from the environment in [lo, 2^30), else dflt.
int env_int(const char* name, int dflt, int lo = 1) {
    const char* v = std::getenv(name);
    if (!v || !*v) return dflt;
    char* end = nullptr;
    long x = std::strtol(v, &end, 10);
    return (end && *end == '\0' && x >= lo && x < (1 << 30)) ? (int)x : dflt;
}

// Bytes of one dispatched element (design page §3.7: the dtype is a property of
// the transport; fp8 and fp4x2 are both one byte, fp4x2 holding a packed pair).
int payload_size(int dtype) { return dtype == EP_FP32 ? 4 : dtype == EP_BF16 ? 2 : 1; }

// The combine leg reduces, so it takes no byte type: float32 for an fp32 plan,
// bf16 otherwise, with 2 * hiddenDim elements for fp4x2 (the unpacked count).
int combine_dtype(int dtype) { return dtype == EP_FP32 ? EP_FP32 : EP_BF16; }
long long combine_hidden(const EpCfg* c) { return c->dtype == EP_FP4X2 ? 2LL * c->hiddenDim : c->hiddenDim; }
long long combine_row_bytes(const EpCfg* c) {
    return combine_hidden(c) * (combine_dtype(c->dtype) == EP_FP32 ? 4 : 2);
}

// The validity rules of the design page §3.5 (EpCfgIsValid / MakeEpCfg) and
// the dtype rule of §3.7, plus the int32 index range of this build.
int check_cfg(const EpCfg* c) {
    if (!c) return fail(EP_ERR_INVALID, "cfg is NULL");
    if (c->worldSize < 1 || c->worldSize > ep::kMaxWorld)
        return fail(EP_ERR_INVALID, "worldSize %d outside 1..%d (one destination per warp lane)",
                    c->worldSize, ep::kMaxWorld);
    if (c->numExpertPerToken < 1 || c->numExpertPerToken > ep::kMaxTopk)
        return fail(EP_ERR_INVALID, "numExpertPerToken %d outside 1..%d (one topk entry per warp lane)",
                    c->numExpertPerToken, ep::kMaxTopk);
    if (c->hiddenDim < 1) return fail(EP_ERR_INVALID, "hiddenDim %d < 1", c->hiddenDim);
    if (c->maxTokPerRank < 1) return fail(EP_ERR_INVALID, "maxTokPerRank %d < 1", c->maxTokPerRank);
    if (c->numExpertPerRank < 1)
        return fail(EP_ERR_INVALID, "numExpertPerRank %d < 1", c->numExpertPerRank);
    if ((long long)c->worldSize * c->numExpertPerRank > (1LL << 30))
        return fail(EP_ERR_INVALID, "too many experts");
    if (c->useWeights != 0 && c->useWeights != 1)
        return fail(EP_ERR_INVALID, "useWeights must be 0 or 1, got %d", c->useWeights);
    if (c->dtype < EP_BF16 || c->dtype > EP_FP4X2) return fail(EP_ERR_INVALID, "unknown dtype %d", c->dtype);
    const long long rowBytes = (long long)c->hiddenDim * payload_size(c->dtype);
    if (rowBytes % 16 != 0)
        return fail(EP_ERR_INVALID, "token bytes %lld (hiddenDim * %d) not a multiple of 16", rowBytes,
                    payload_size(c->dtype));
    const long long G = (long long)c->worldSize * c->maxTokPerRank;
    if (G > (1LL << 30)) return fail(EP_ERR_INVALID, "worldSize*maxTokPerRank too large");
    if (c->maxRecv < 0) return fail(EP_ERR_INVALID, "maxRecv %d < 0", c->maxRecv);
    const long long maxRecv = c->maxRecv == 0 ? G : c->maxRecv;
    if (maxRecv < G)
        return fail(EP_ERR_INVALID,
                    "maxRecv %lld does not cover the worst case worldSize*maxTokPerRank = %lld", maxRecv, G);
    if ((long long)c->worldSize * maxRecv > (1LL << 31) - 1)
        return fail(EP_ERR_INVALID, "worldSize*maxRecv exceeds the int32 flat index");
    return EP_OK;
}

struct Geometry {
    int chunkBytes, chunkStride, numChunks;
    int scatterWarps, scatterStages;
    int combineWarps;
};

// Copy engines and stages: three engines (warps) per block for rows of 8 KB
// and more, two otherwise, each with as many row-sized stages as fit in about
// 215 KB of shared memory (at most 8; two engines when fewer than 4 stages
// would fit; rows above 32 KB are copied in pieces of <= 16 KB). On B200 at
// 14 KB rows, 3 x 5 with one engine sitting out at a high fan-out matches 2 x 7
// on uniform routing (472 us) and beats it by 12% on skewed routing (295 vs
// 335 us); 1 x 14 is far slower (one issuing thread per SM).
Geometry pick_geometry(const EpCfg* c, bool use_env) {
    Geometry g{};
    const long long rowBytes = (long long)c->hiddenDim * payload_size(c->dtype);
    int chunk;
    if (rowBytes <= 32768) {
        chunk = (int)rowBytes;
    } else {
        const long long pieces = (rowBytes + 16383) / 16384;
        chunk = (int)(((rowBytes + pieces - 1) / pieces + 15) & ~15LL);
    }
    if (use_env) chunk = std::min<long long>(rowBytes, env_int("EP_SCATTER_CHUNK", chunk) & ~15);
    if (chunk < 16) chunk = 16;
    g.chunkBytes = chunk;
    g.chunkStride = (chunk + 127) & ~127;
    g.numChunks = (int)((rowBytes + chunk - 1) / chunk);
    // Rows of 8 KB and more: one block per SM of about 215 KB, with a third
    // engine that sits out at a high fan-out (see copy_engine). Rows between
    // 4 and 8 KB: two engines per block and two blocks per SM, each within
    // about 110 KB (an SM has 228 KB, and each block also holds its static
    // shared memory and 1 KB the system keeps). B200, fp8 rows of 7 KB at the
    // main workload: 8 stages left one block per SM once the static shared
    // memory grew (419 us), 7 stages keep two (245 us); 3 x 4, 3 x 5 and 2 x 6
    // measured 246-248 us. Rows of at most 4 KB: three engines of 5 stages, as
    // many blocks as fit an SM (per-token work weighs more against small rows):
    // fp4x2 rows of 3.5 KB at the main workload 135.4 vs 160.9 us with 2 x 8
    // (5 x 5 136.3, 4 x 5 142.1, 8 x 3 144.9), the ct = 1 workload's 4 KB rows
    // 14.3 vs 15.3 us.
    int warps = g.chunkStride >= 8192 ? 3 : 2;
    const int budget = 215 * 1024;
    int stages = (warps == 3 ? budget : 110 * 1024) / (warps * g.chunkStride);
    if (g.chunkStride <= 4096) {
        warps = 3;
        stages = 5;
    }
    if (stages < 4) {
        warps = 2;
        stages = budget / (warps * g.chunkStride);
    }
    if (stages < 2) {
        warps = std::max(1, budget / (2 * g.chunkStride));
        stages = 2;
    }
    stages = std::min(stages, 8);
    if (use_env) {
        warps = std::min(env_int("EP_SCATTER_WARPS", warps), ep::kMaxScatterWarps);
        stages = std::max(2, std::min(env_int("EP_SCATTER_STAGES", stages), 16));
    }
    g.scatterWarps = warps;
    g.scatterStages = stages;
    g.combineWarps = use_env ? std::min(env_int("EP_COMBINE_WARPS", 8), ep::kMaxCombineWarps) : 8;
    return g;
}

// The fused dispatch (dispatch_fused, EP_DISPATCH_FUSED=1): one launch in
// which every block routes its own share of the batch and copies it, for
// plans where no block owns more than kFusedMaxOwn tokens. Taken only on
// request: on B200 it measured about as fast as route_count + scatter_rows at
// the 512-token workload (28.4-28.9 vs 29.7 us) and slower where a few
// present tokens cluster (ct = 8 of 512 tokens a rank: 17.7 vs 15.2 us),
// since a block's present tokens all go through that block's engines.
bool want_fused() {
    const char* v = std::getenv("EP_DISPATCH_FUSED");
    return v && std::strcmp(v, "1") == 0;
}

}  // namespace

namespace ep {
bool combine_wide_loads(long long outBytes, long long rowBytes);  // defined below
}

namespace {
// The combine reads y in 32-byte loads when its output, W*T combine rows, is
// at least 192 MiB and the rows are a multiple of 32 bytes (a call whose y is
// not 32-byte aligned takes 16-byte loads). B200, W=8, topk 8, output size ->
// 16- vs 32-byte loads: 67 MB 72.7 vs 76.6 us, 117 MB 128.7 vs 136.1, 134 MB
// (h=2048, 32768 tokens) 135.5 vs 140.0 and (h=4096, 16384 tokens) 139.9 vs
// 144.8; 235 MB 235.4 vs 233.9, 268 MB 262.8 vs 259.6, 470 MB 454.0 vs 442.8
// (h=7168) and 464.4 vs 452.5 (h=14336), 940 MB 902.5 vs 872.7.
// EP_COMBINE_WIDE=0/1 overrides the size rule.
bool combine_wide(const EpCfg* c) {
    return ep::combine_wide_loads((long long)c->worldSize * c->maxTokPerRank * combine_row_bytes(c),
                                  combine_row_bytes(c));
}

void fill_info(const EpCfg* c, const Geometry& geo, EpPlanInfo* info) {
    std::memset(info, 0, sizeof *info);
    const long long G = (long long)c->worldSize * c->maxTokPerRank;
    const int maxRecv = c->maxRecv == 0 ? (int)G : c->maxRecv;
    const int M = 3 + c->numExpertPerToken;
    info->maxRecv = maxRecv;
    info->metaFields = M;
    info->rowBytes = (long long)c->hiddenDim * payload_size(c->dtype);
    info->tokenBytes = G * info->rowBytes;
    info->recvXBytes = (long long)c->worldSize * maxRecv * info->rowBytes;
    info->combineDtype = combine_dtype(c->dtype);
    info->combineHidden = (int32_t)combine_hidden(c);
    info->combineRowBytes = combine_row_bytes(c);
    info->yBytes = (long long)c->worldSize * maxRecv * info->combineRowBytes;
    info->outBytes = G * info->combineRowBytes;
    info->recvMetaBytes = (long long)c->worldSize * maxRecv * M * 4;
    info->countTile = ep::kCountTile;
    info->numTiles = (int)((G + ep::kCountTile - 1) / ep::kCountTile);
    info->scratchBytes = (long long)ep::scratch_layout(G, c->worldSize, info->numTiles).total;
    info->scatterWarps = geo.scatterWarps;
    info->scatterStages = geo.scatterStages;
    info->scatterChunkBytes = geo.chunkBytes;
    info->scatterMode = 0;  // TMA bulk copies staged in shared memory
    info->scatterPend = 1;  // one item's bulk stores left draining when a stage refills
    info->combineWarps = geo.combineWarps;
    info->device = -1;
    info->combineLoadBytes = combine_wide(c) ? 32 : 16;
}

}  // namespace

namespace ep {
void set_last_error(const char* msg) { std::snprintf(g_last_error, sizeof g_last_error, "%s", msg); }

bool combine_wide_loads(long long outBytes, long long rowBytes) {
    if (rowBytes % 32 != 0) return false;
    const int env = env_int("EP_COMBINE_WIDE", -1, 0);
    if (env >= 0) return env != 0;
    return outBytes >= (192LL << 20);
}

int fail_code(int code, const char* msg) { return fail(code, "%s", msg); }

int cfg_valid(const EpCfg* cfg) { return check_cfg(cfg); }

// The split dispatch's copy geometry of a plan of cfg on the current device,
// with route_count's last block scanning the tile counts (no tile table in
// the scatter's shared memory), and the combine's grid.
int copy_geometry(const EpCfg* cfg, CopyGeometry* out) {
    int dev = 0, sms = 0, smemOptin = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&smemOptin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
        return cuda_fail(e, "device attributes");
    Geometry geo = pick_geometry(cfg, true);
    const size_t limit = (size_t)smemOptin - kStaticSmemReserve;
    size_t smem = scatter_smem_bytes(geo.scatterWarps, geo.scatterStages, geo.chunkStride);
    while (smem > limit && geo.scatterStages > 2)
        smem = scatter_smem_bytes(geo.scatterWarps, --geo.scatterStages, geo.chunkStride);
    while (smem > limit && geo.scatterWarps > 1)
        smem = scatter_smem_bytes(--geo.scatterWarps, geo.scatterStages, geo.chunkStride);
    if (smem > limit) return fail(EP_ERR_INVALID, "row piece of %d bytes does not fit shared memory", geo.chunkBytes);
    int sPerSm = 0, cPerSm = 0;
    if ((e = scatter_set_smem(smem)) != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(scatter smem)");
    if ((e = scatter_blocks_per_sm(geo.scatterWarps, smem, &sPerSm)) != cudaSuccess ||
        (e = combine_blocks_per_sm(geo.combineWarps, cfg->dtype == EP_FP32, &cPerSm)) != cudaSuccess)
        return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (sPerSm < 1 || cPerSm < 1) return fail(EP_ERR_INVALID, "kernel geometry does not fit one SM");
    out->chunkBytes = geo.chunkBytes;
    out->chunkStride = geo.chunkStride;
    out->numChunks = geo.numChunks;
    out->warps = geo.scatterWarps;
    out->stages = geo.scatterStages;
    out->blocks = env_int("EP_SCATTER_BLOCKS", sms * sPerSm);
    out->smem = smem;
    out->combineWarps = geo.combineWarps;
    out->combineBlocks = env_int("EP_COMBINE_BLOCKS", sms * cPerSm);
    out->numSMs = sms;
    out->device = dev;
    return EP_OK;
}
}  // namespace ep

extern "C" {

const char* ep_last_error(void) { return g_last_error; }

int ep_cfg_check(const EpCfg* cfg) {
    try {
        g_last_error[0] = '\0';
        return check_cfg(cfg);
    } catch (...) {
        return fail(EP_ERR_INVALID, "unexpected exception");
    }
}

int ep_plan_query(const EpCfg* cfg, EpPlanInfo* info) {
    try {
        if (!info) return fail(EP_ERR_INVALID, "info is NULL");
        int rc = check_cfg(cfg);
        if (rc) return rc;
        const Geometry geo = pick_geometry(cfg, false);
        fill_info(cfg, geo, info);
        const int sms = 148;  // B200
        // Blocks per SM: the SM's 228 KB over the block's shared memory, its
        // static shared memory and the 1 KB the system keeps per block.
        const size_t perBlock = ep::scatter_smem_bytes(geo.scatterWarps, std::max(geo.scatterStages, 1),
                                                       geo.chunkStride) + ep::kStaticSmemReserve + 1024;
        info->scatterBlocks = sms * std::max(1, (int)((228 * 1024) / perBlock));
        info->combineBlocks = sms * 2;
        const long long G = (long long)cfg->worldSize * cfg->maxTokPerRank;
        const int fusedBlocks = (int)std::min<long long>(info->scatterBlocks, G);
        if (want_fused() && (G + fusedBlocks - 1) / fusedBlocks <= ep::kFusedMaxOwn) {
            info->dispatchFused = 1;
            info->scatterBlocks = fusedBlocks;
            info->scratchBytes = (long long)ep::scratch_layout(G, cfg->worldSize, info->numTiles, fusedBlocks).total;
        }
        return EP_OK;
    } catch (...) {
        return fail(EP_ERR_INVALID, "unexpected exception");
    }
}

EpPlan* ep_plan_create(const EpCfg* cfg) {
    EpPlan* plan = nullptr;
    try {
        if (check_cfg(cfg) != EP_OK) return nullptr;
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) {
            cuda_fail(e, "cudaGetDevice");
            return nullptr;
        }
        int sms = 0, smemOptin = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&smemOptin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
                cudaSuccess) {
            cuda_fail(e, "cudaDeviceGetAttribute");
            return nullptr;
        }
        Geometry geo = pick_geometry(cfg, true);
        size_t smem = 0, baseSmem = 0, baseOffset = 0, engineOffset = 0;
        // Batches above kDenseMinTokens tokens take route_count in its
        // large-batch form with the dense copy path: on B200 the main
        // workload's dispatch measured 470 us that way against 478 us with
        // the sparse-batch machinery (present-token column, scatter-side
        // scan), which pays off only for small batches (ct = 1: 15.3 vs
        // 17.4 us). EP_DISPATCH_DENSE=0/1 overrides.
        constexpr long long kDenseMinTokens = 16384;
        const long long Gtok = (long long)cfg->worldSize * cfg->maxTokPerRank;
        const int denseEnv = env_int("EP_DISPATCH_DENSE", -1, 0);
        const bool dense = denseEnv >= 0 ? denseEnv != 0 : Gtok > kDenseMinTokens;
        {
            // The scatter scans route_count's tile counts itself when they
            // fit a few KB of shared memory (route_count then ends without a
            // last-block scan). Shared memory:
            // the tile bases (if any) first, then the copy engines.
            const int numTiles =
                (int)(((long long)cfg->worldSize * cfg->maxTokPerRank + ep::kCountTile - 1) / ep::kCountTile);
            const size_t bs = ep::scatter_base_smem_bytes(numTiles, cfg->worldSize);
            const char* scanEnv = std::getenv("EP_SCATTER_SCAN");
            const bool scanInRoute = scanEnv && std::strcmp(scanEnv, "route") == 0;
            if (!scanInRoute && !dense && bs <= ep::kMaxBaseSmemBytes) baseSmem = bs;
            const size_t limit = (size_t)smemOptin - ep::kStaticSmemReserve;
            auto engines = [&]() {
                return ep::scatter_smem_bytes(geo.scatterWarps, geo.scatterStages, geo.chunkStride);
            };
            // The table must not cost a block per SM (7 KB rows: 2 blocks of
            // 8 stages fit an SM without it, 1 with it).
            if (baseSmem > 0) {
                const size_t eng = engines();
                int with = 0, without = 0;
                if ((e = ep::scatter_set_smem(std::min(limit, eng + baseSmem + 1024))) != cudaSuccess ||
                    (e = ep::scatter_blocks_per_sm(geo.scatterWarps, std::min(limit, eng), &without)) !=
                        cudaSuccess ||
                    (e = ep::scatter_blocks_per_sm(geo.scatterWarps, std::min(limit, eng + baseSmem), &with)) !=
                        cudaSuccess) {
                    cuda_fail(e, "scatter occupancy");
                    return nullptr;
                }
                if (with < without) baseSmem = 0;
            }
            smem = baseSmem + engines();
            while (smem > limit && geo.scatterStages > 2) {
                --geo.scatterStages;
                smem = baseSmem + engines();
            }
            while (smem > limit && geo.scatterWarps > 1) {
                --geo.scatterWarps;
                smem = baseSmem + engines();
            }
            if (smem > limit) {
                fail(EP_ERR_INVALID, "row piece of %d bytes does not fit shared memory", geo.chunkBytes);
                return nullptr;
            }
            baseOffset = 0;
            engineOffset = baseSmem;
            if ((e = ep::scatter_set_smem(smem)) != cudaSuccess) {
                cuda_fail(e, "cudaFuncSetAttribute(scatter smem)");
                return nullptr;
            }
        }
        int sPerSm = 0, cPerSm = 0;
        if ((e = ep::scatter_blocks_per_sm(geo.scatterWarps, smem, &sPerSm)) != cudaSuccess ||
            (e = ep::combine_blocks_per_sm(geo.combineWarps, cfg->dtype == EP_FP32, &cPerSm)) != cudaSuccess) {
            cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
            return nullptr;
        }
        if (sPerSm < 1 || cPerSm < 1) {
            fail(EP_ERR_INVALID, "kernel geometry does not fit one SM");
            return nullptr;
        }

        plan = new (std::nothrow) EpPlan();
        if (!plan) {
            fail(EP_ERR_NOMEM, "host allocation failed");
            return nullptr;
        }
        plan->cfg = *cfg;
        fill_info(cfg, geo, &plan->info);
        plan->device = dev;
        plan->info.device = dev;
        plan->info.numSMs = sms;
        plan->info.scatterBlocks = env_int("EP_SCATTER_BLOCKS", sms * sPerSm);
        // The fused dispatch, on request (want_fused).
        plan->fused = false;
        {
            const long long G = (long long)cfg->worldSize * cfg->maxTokPerRank;
            int blocks = plan->info.scatterBlocks;
            // Copy engines: a block's present tokens all go through its own
            // engines, so where rows are small there are more of them (with at
            // least 3 stages each, in the split scatter's shared memory),
            // unless the geometry is set by hand.
            int fEngines = geo.scatterWarps, fStages = geo.scatterStages;
            if (!std::getenv("EP_SCATTER_WARPS") && !std::getenv("EP_SCATTER_STAGES")) {
                const long long budget = (long long)geo.scatterWarps * geo.scatterStages * geo.chunkStride;
                fEngines = (int)std::max<long long>(geo.scatterWarps,
                                                    std::min<long long>(ep::kFusedWarps, budget / (3LL * geo.chunkStride)));
                fStages = (int)std::max<long long>(2, std::min<long long>(8, budget / ((long long)fEngines * geo.chunkStride)));
            }
            if (want_fused() && fEngines <= ep::kFusedWarps) {
                // The grid: the scatter's, at most one block a token, at most
                // what fits the SMs at once (the routing area may cost a block
                // per SM, which changes the tokens a block owns: try again).
                const size_t limit = (size_t)smemOptin - ep::kStaticSmemReserve;
                blocks = (int)std::min<long long>(blocks, G);
                for (int attempt = 0; attempt < 3 && blocks >= 1; ++attempt) {
                    const int own = (int)((G + blocks - 1) / blocks);
                    if (own > ep::kFusedMaxOwn) break;
                    const size_t area =
                        ep::fused_layout(own, cfg->worldSize, ep::kFusedWarps, cfg->numExpertPerToken).total;
                    int stages = fStages;
                    size_t lsm = area + ep::scatter_smem_bytes(fEngines, stages, geo.chunkStride);
                    while (lsm > limit && stages > 2)
                        lsm = area + ep::scatter_smem_bytes(fEngines, --stages, geo.chunkStride);
                    if (lsm > limit) break;
                    int per = 0;
                    if ((e = ep::fused_set_smem(cfg->worldSize, cfg->numExpertPerToken, lsm)) != cudaSuccess ||
                        (e = ep::fused_blocks_per_sm(cfg->worldSize, cfg->numExpertPerToken, lsm, &per)) !=
                            cudaSuccess) {
                        cuda_fail(e, "dispatch_fused set-up");
                        delete plan;
                        return nullptr;
                    }
                    if (per < 1) break;
                    if (blocks > sms * per) {
                        blocks = sms * per;
                        continue;
                    }
                    plan->fused = true;
                    plan->fusedSmem = lsm;
                    plan->fusedEngineOffset = area;
                    plan->fusedOwn = own;
                    plan->fusedBlocks = blocks;
                    plan->info.scatterBlocks = blocks;
                    plan->info.scatterWarps = fEngines;
                    plan->info.scatterStages = stages;
                    break;
                }
            }
        }
        plan->info.dispatchFused = plan->fused ? 1 : 0;
        plan->fanoutSwitch = env_int("EP_SCATTER_FANOUT_SWITCH", 375, 0);
        // Test hook for the failure path: the fused dispatch's wait for the
        // earlier blocks' totals can never complete, so the blocks give up
        // after their bounded wait and report EP_DEVERR_TIMEOUT.
        if (const char* t = std::getenv("EP_TEST_UNREACHABLE_BARRIER"))
            plan->barrierSlack = std::strcmp(t, "1") == 0 ? 1u : 0u;
        // Test hook of the bounds-checking build: check the receive buffers
        // against fewer rows than they have, so that the checks must fire.
        plan->boundsRows = std::min(env_int("EP_TEST_BOUNDS_ROWS", plan->info.maxRecv), plan->info.maxRecv);
        plan->info.combineBlocks = env_int("EP_COMBINE_BLOCKS", sms * cPerSm);
        plan->scatterSmem = smem;
        plan->dense = dense;
        plan->baseSmem = baseSmem;
        plan->baseOffset = baseOffset;
        plan->engineOffset = engineOffset;
        plan->G = cfg->worldSize * cfg->maxTokPerRank;
        plan->maxRecv = plan->info.maxRecv;

        const ep::ScratchLayout L =
            ep::scratch_layout(plan->G, cfg->worldSize, plan->info.numTiles, plan->fused ? plan->fusedBlocks : 0);
        plan->info.scratchBytes = (long long)L.total;
        const size_t total = L.total;
        if ((e = cudaMalloc(&plan->scratch, total)) != cudaSuccess) {
            cuda_fail(e, "cudaMalloc(plan scratch)");
            plan->scratch = nullptr;
            ep_plan_destroy(plan);
            return nullptr;
        }
        if ((e = cudaMemset(plan->scratch, 0, total)) != cudaSuccess) {
            cuda_fail(e, "cudaMemset(plan scratch)");
            ep_plan_destroy(plan);
            return nullptr;
        }
        char* base = static_cast<char*>(plan->scratch);
        plan->route = reinterpret_cast<int2*>(base + L.route);
        plan->tok_mask = reinterpret_cast<uint32_t*>(base + L.tok_mask);
        plan->tile_cnt = reinterpret_cast<int32_t*>(base + L.tile_cnt);
        plan->tile_base = reinterpret_cast<int32_t*>(base + L.tile_base);
        plan->ticket = reinterpret_cast<uint32_t*>(base + L.ticket);
        plan->work = reinterpret_cast<int32_t*>(base + L.work);
        plan->ptotal = reinterpret_cast<int32_t*>(base + L.ptotal);
        plan->cwork = reinterpret_cast<int32_t*>(base + L.cwork);
        plan->cdone = reinterpret_cast<uint32_t*>(base + L.cdone);
        plan->err = reinterpret_cast<int32_t*>(base + L.err);
        plan->fused_agg = reinterpret_cast<unsigned long long*>(base + L.fused_agg);
        plan->fused_epoch = reinterpret_cast<unsigned*>(base + L.fused_epoch);
        plan->fused_done = reinterpret_cast<unsigned*>(base + L.fused_done);
        plan->dispatched = false;
        g_last_error[0] = '\0';
        return plan;
    } catch (...) {
        fail(EP_ERR_INVALID, "unexpected exception");
        if (plan) ep_plan_destroy(plan);
        return nullptr;
    }
}

void ep_plan_destroy(EpPlan* plan) {
    if (!plan) return;
    if (plan->scratch) cudaFree(plan->scratch);
    delete plan;
}

int ep_plan_info(const EpPlan* plan, EpPlanInfo* info) {
    if (!plan || !info) return fail(EP_ERR_INVALID, "plan or info is NULL");
    *info = plan->info;
    return EP_OK;
}

static int check_device(const EpPlan* plan) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev != plan->device)
        return fail(EP_ERR_DEVICE, "current device %d is not the plan's device %d", dev, plan->device);
    return EP_OK;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static int dispatch_impl(EpPlan* plan, const void* x, const int32_t* topk_idx, const float* topk_w,
                         const void* scales, int32_t scaleWords, void* recv_x, int32_t* recv_meta,
                         void* recv_scales, int32_t* recv_count, void* stream);

int ep_dispatch(EpPlan* plan, const void* x, const int32_t* topk_idx, const float* topk_w,
                void* recv_x, int32_t* recv_meta, int32_t* recv_count, void* stream) {
    return dispatch_impl(plan, x, topk_idx, topk_w, nullptr, 0, recv_x, recv_meta, nullptr, recv_count,
                         stream);
}

int ep_dispatch_scaled(EpPlan* plan, const void* x, const int32_t* topk_idx, const float* topk_w,
                       const void* scales, int32_t scaleWords, void* recv_x, int32_t* recv_meta,
                       void* recv_scales, int32_t* recv_count, void* stream) {
    if (scaleWords < 1 || scaleWords > EP_MAX_SCALE_WORDS)
        return fail(EP_ERR_INVALID, "scaleWords %d outside 1..%d", scaleWords, EP_MAX_SCALE_WORDS);
    if (!scales || !recv_scales) return fail(EP_ERR_INVALID, "scales or recv_scales is NULL");
    if (!aligned(scales, 4) || !aligned(recv_scales, 4))
        return fail(EP_ERR_ALIGN, "scales and recv_scales must be 4-byte aligned");
    return dispatch_impl(plan, x, topk_idx, topk_w, scales, scaleWords, recv_x, recv_meta, recv_scales,
                         recv_count, stream);
}

static int dispatch_impl(EpPlan* plan, const void* x, const int32_t* topk_idx, const float* topk_w,
                         const void* scales, int32_t scaleWords, void* recv_x, int32_t* recv_meta,
                         void* recv_scales, int32_t* recv_count, void* stream) {
    try {
        if (!plan) return fail(EP_ERR_INVALID, "plan is NULL");
        if (!x || !topk_idx || !recv_x || !recv_meta || !recv_count)
            return fail(EP_ERR_INVALID, "a required buffer is NULL");
        if (plan->cfg.useWeights && !topk_w)
            return fail(EP_ERR_INVALID, "topk_w is NULL but useWeights is 1");
        if (!aligned(x, 16) || !aligned(recv_x, 16))
            return fail(EP_ERR_ALIGN, "x and recv_x must be 16-byte aligned");
        if (!aligned(topk_idx, 4) || !aligned(recv_meta, 4) || !aligned(recv_count, 4) ||
            (topk_w && !aligned(topk_w, 4)))
            return fail(EP_ERR_ALIGN, "topk_idx, topk_w, recv_meta, recv_count must be 4-byte aligned");
        int rc = check_device(plan);
        if (rc) return rc;
        const EpCfg& c = plan->cfg;
        cudaStream_t s = static_cast<cudaStream_t>(stream);

        ep::RouteParams rp{};
        rp.idx = topk_idx;
        rp.w = c.useWeights ? topk_w : nullptr;
        rp.route = plan->route;
        rp.tok_mask = plan->tok_mask;
        rp.tile_cnt = plan->tile_cnt;
        rp.tile_base = plan->tile_base;
        rp.recv_count = recv_count;
        rp.ticket = plan->ticket;
        rp.work = plan->work;
        rp.ptotal = plan->ptotal;
        rp.lastScan = plan->baseSmem == 0 ? 1 : 0;
        rp.err = plan->err;
        rp.G = plan->G;
        rp.W = c.worldSize;
        rp.k = c.numExpertPerToken;
        rp.nEpr = c.numExpertPerRank;
        rp.E = c.worldSize * c.numExpertPerRank;
        rp.numTiles = plan->info.numTiles;
        rp.maxRecv = plan->maxRecv;
        rp.useWeights = c.useWeights;
        cudaError_t e = cudaSuccess;

        ep::ScatterParams sp{};
        sp.x = static_cast<const uint8_t*>(x);
        sp.idx = topk_idx;
        sp.route = plan->route;
        sp.tok_mask = plan->tok_mask;
        sp.tile_base = plan->tile_base;
        sp.work = plan->work;
        sp.recv_x = static_cast<uint8_t*>(recv_x);
        sp.recv_meta = recv_meta;
        sp.err = plan->err;
        sp.rowBytes = plan->info.rowBytes;
        sp.G = plan->G;
        sp.W = c.worldSize;
        sp.k = c.numExpertPerToken;
        sp.nEpr = c.numExpertPerRank;
        sp.E = c.worldSize * c.numExpertPerRank;
        sp.T = c.maxTokPerRank;
        sp.maxRecv = plan->maxRecv;
        sp.M = plan->info.metaFields;
        sp.chunkBytes = plan->info.scatterChunkBytes;
        sp.chunkStride = (sp.chunkBytes + 127) & ~127;
        sp.numChunks = (int)((sp.rowBytes + sp.chunkBytes - 1) / sp.chunkBytes);
        sp.stages = plan->info.scatterStages;
        sp.recv_count = recv_count;
        sp.fanoutSwitch = plan->fanoutSwitch;
        sp.scales = static_cast<const uint32_t*>(scales);
        sp.recv_scales = static_cast<uint32_t*>(recv_scales);
        sp.scaleWords = scaleWords;
        sp.boundsRows = plan->boundsRows;
        if (plan->fused) {
            // One launch: each block routes its own tokens, adds up the earlier blocks' totals, copies its own.
            const int nEpr = c.numExpertPerRank;
            sp.w = c.useWeights ? topk_w : nullptr;
            sp.useWeights = c.useWeights;
            sp.nEprShift = (nEpr & (nEpr - 1)) == 0 ? __builtin_ctz((unsigned)nEpr) : -1;
            sp.fusedOwn = plan->fusedOwn;
            sp.fusedEngines = plan->info.scatterWarps;
            sp.engineOffset = (int)plan->fusedEngineOffset;
            sp.fused_agg = plan->fused_agg;
            sp.fused_epoch = plan->fused_epoch;
            sp.fused_done = plan->fused_done;
            sp.barrierSlack = plan->barrierSlack;
            // One row load per copy engine before the look-back: B200, one run at the
            // 512-token workload, none 27.7 us, one 27.1, two 28.8, all (three) 28.7:
            // more rows in flight delay the look-back's loads behind them.
            sp.earlyIssue = 1;
            e = ep::launch_dispatch_fused(sp, plan->fusedBlocks, plan->fusedSmem, s);
            if (e != cudaSuccess) return cuda_fail(e, "launch dispatch_fused");
            plan->dispatched = true;
            return EP_OK;
        }
        e = ep::launch_route_count(rp, plan->dense, s);
        if (e != cudaSuccess) return cuda_fail(e, "launch route_count");
        sp.baseShift = 8;  // route_count's 256-token tiles
        sp.baseStride = plan->dense ? c.worldSize : c.worldSize + 1;
        sp.tile_cnt = plan->tile_cnt;
        sp.numTiles = plan->info.numTiles;
        sp.baseSmemBytes = (int)plan->baseSmem;
        sp.baseOffset = (int)plan->baseOffset;
        sp.engineOffset = (int)plan->engineOffset;
        sp.ptotal = plan->dense ? nullptr : plan->ptotal;  // dense: every token counts as present
        e = ep::launch_scatter_rows(sp, plan->dense, plan->info.scatterBlocks, plan->info.scatterWarps,
                                    plan->scatterSmem, s);
        if (e != cudaSuccess) return cuda_fail(e, "launch scatter_rows");
        plan->dispatched = true;
        return EP_OK;
    } catch (...) {
        return fail(EP_ERR_INVALID, "unexpected exception");
    }
}

int ep_combine(EpPlan* plan, const void* y, void* out, void* stream) {
    try {
        if (!plan) return fail(EP_ERR_INVALID, "plan is NULL");
        if (!y || !out) return fail(EP_ERR_INVALID, "y or out is NULL");
        if (!aligned(y, 16) || !aligned(out, 16))
            return fail(EP_ERR_ALIGN, "y and out must be 16-byte aligned");
        if (!plan->dispatched) return fail(EP_ERR_STATE, "combine before any dispatch on this plan");
        int rc = check_device(plan);
        if (rc) return rc;
        ep::CombineParams cp{};
        cp.y = static_cast<const uint8_t*>(y);
        cp.route = plan->route;
        cp.out = static_cast<uint8_t*>(out);
        cp.work = plan->cwork;
        cp.done = plan->cdone;
        cp.rowBytes = plan->info.combineRowBytes;
        cp.G = plan->G;
        cp.W = plan->cfg.worldSize;
        cp.maxRecv = plan->maxRecv;
        cp.err = plan->err;
        cp.yBytes = plan->info.yBytes;
        const bool wide = plan->info.combineLoadBytes == 32 && aligned(y, 32);
        cudaError_t e = ep::launch_combine(cp, plan->info.combineDtype == EP_FP32, wide, plan->info.combineBlocks,
                                           plan->info.combineWarps,
                                           static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "launch combine");
        return EP_OK;
    } catch (...) {
        return fail(EP_ERR_INVALID, "unexpected exception");
    }
}

int ep_plan_check_error(EpPlan* plan) {
    if (!plan) return fail(EP_ERR_INVALID, "plan is NULL");
    int rc = check_device(plan);
    if (rc) return rc;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    int32_t word = 0;
    if ((e = cudaMemcpy(&word, plan->err, sizeof word, cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "cudaMemcpy(error word)");
    if ((e = cudaMemset(plan->err, 0, sizeof word)) != cudaSuccess) return cuda_fail(e, "cudaMemset");
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    return word;
}

}  // extern "C"
