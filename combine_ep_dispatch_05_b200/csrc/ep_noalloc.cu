// ep_noalloc.cu -- ep_dispatch_noalloc: dispatch without a plan and without
// any device allocation.
//
// Some callers cannot call cudaMalloc at the point where they dispatch: code
// that runs while a memory pool must not grow (a serving loop under a fixed
// memory budget), code inside allocator or driver callbacks where allocating
// would re-enter the allocator, or embedders whose runtime owns every device
// allocation. For them this entry point takes its scratch memory (routing
// table, per-tile counts and bases, tile ticket, error word) from one
// file-scope __device__ array of EP_NOALLOC_SCRATCH_BYTES bytes instead of a
// plan's cudaMalloc'd scratch. The array exists on every device that loads the
// library and stays there until the process exits.
//
// It runs the same route_count and scatter_rows kernels as ep_dispatch, so its
// outputs are identical to a plan's dispatch of the same configuration.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "ep.h"
#include "ep_internal.h"

namespace {

// The scratch of every ep_dispatch_noalloc call on this device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[EP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct DeviceSetup {
    bool ready = false;
    unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch
    int numSMs = 0;
    int smemOptin = 0;
};

std::mutex g_setup_mutex;
DeviceSetup g_setup[kMaxDevices];

// Failures are reported like every other entry point: a negative code, and
// the reason in ep_last_error().
int noalloc_fail(int code, const char* fmt, ...) {
    char msg[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(msg, sizeof msg, fmt, ap);
    va_end(ap);
    ep::set_last_error(msg);
    return code;
}

// Once per device, with that device current: the device address of the
// scratch array (the host-side symbol is only a stand-in for it) and the
// device limits the launch geometry needs.
int setup_device(int dev, DeviceSetup* out) {
    if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(EP_ERR_DEVICE, "device %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    DeviceSetup& s = g_setup[dev];
    if (!s.ready) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return noalloc_fail(EP_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        int sms = 0, smem = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
            return noalloc_fail(EP_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        s.scratch = static_cast<unsigned char*>(p);
        s.numSMs = sms;
        s.smemOptin = smem;
        s.ready = true;
    }
    *out = s;
    return EP_OK;
}

}  // namespace

extern "C" int ep_dispatch_noalloc(const EpCfg* cfg, const void* x, const int32_t* topk_idx,
                                   const float* topk_w, void* recv_x, int32_t* recv_meta,
                                   int32_t* recv_count, void* stream) {
    try {
        ep::set_last_error("");
        int rc = ep_cfg_check(cfg);
        if (rc) return noalloc_fail(rc, "%s", ep_last_error());
        if (!x || !topk_idx || !recv_x || !recv_meta || !recv_count)
            return noalloc_fail(EP_ERR_INVALID, "a required buffer is NULL");
        if (cfg->useWeights && !topk_w) return noalloc_fail(EP_ERR_INVALID, "topk_w is NULL but useWeights is 1");
        if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(recv_x)) % 16 != 0)
            return noalloc_fail(EP_ERR_ALIGN, "x and recv_x must be 16-byte aligned");
        // The same 4-byte rule as ep_dispatch: the kernels load and store these as int32 / float.
        if ((reinterpret_cast<uintptr_t>(topk_idx) | reinterpret_cast<uintptr_t>(recv_meta) |
             reinterpret_cast<uintptr_t>(recv_count) | reinterpret_cast<uintptr_t>(topk_w)) % 4 != 0)
            return noalloc_fail(EP_ERR_ALIGN, "topk_idx, topk_w, recv_meta, recv_count must be 4-byte aligned");

        // Sizes and geometry of the default plan for this configuration.
        EpPlanInfo info;
        if ((rc = ep_plan_query(cfg, &info)) != EP_OK) return noalloc_fail(rc, "%s", ep_last_error());
        const int W = cfg->worldSize;
        const long long G = (long long)W * cfg->maxTokPerRank;
        const ep::ScratchLayout L = ep::scratch_layout(G, W, info.numTiles);
        const size_t need = L.total;
        if (need > (size_t)EP_NOALLOC_SCRATCH_BYTES)
            return noalloc_fail(EP_ERR_INVALID,
                                "configuration needs %zu bytes of scratch; ep_dispatch_noalloc has %d "
                                "(the routing table alone is worldSize^2 * maxTokPerRank * 8 bytes)",
                                need, (int)EP_NOALLOC_SCRATCH_BYTES);

        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return noalloc_fail(EP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
        DeviceSetup ds;
        if ((rc = setup_device(dev, &ds)) != EP_OK) return rc;

        unsigned char* base = ds.scratch;
        int2* route = reinterpret_cast<int2*>(base + L.route);
        uint32_t* tok_mask = reinterpret_cast<uint32_t*>(base + L.tok_mask);
        int32_t* tile_cnt = reinterpret_cast<int32_t*>(base + L.tile_cnt);
        int32_t* tile_base = reinterpret_cast<int32_t*>(base + L.tile_base);
        uint32_t* ticket = reinterpret_cast<uint32_t*>(base + L.ticket);
        int32_t* work = reinterpret_cast<int32_t*>(base + L.work);
        int32_t* ptotal = reinterpret_cast<int32_t*>(base + L.ptotal);
        int32_t* err = reinterpret_cast<int32_t*>(base + L.err);
        cudaStream_t s = static_cast<cudaStream_t>(stream);

        // The scratch keeps whatever the previous call left: the tile ticket
        // and the error word must start at zero.
        if ((e = cudaMemsetAsync(ticket, 0, 512, s)) != cudaSuccess)
            return noalloc_fail(EP_ERR_CUDA, "cudaMemsetAsync(scratch): %s", cudaGetErrorString(e));

        // Scatter geometry: the default plan's engines and stages.
        const int warps = info.scatterWarps;
        int stages = std::max(info.scatterStages, 2);
        const int chunkStride = (info.scatterChunkBytes + 127) & ~127;
        const size_t smemMax = (size_t)ds.smemOptin - ep::kStaticSmemReserve;
        size_t smem = ep::scatter_smem_bytes(warps, stages, chunkStride);
        while (smem > smemMax && stages > 2) smem = ep::scatter_smem_bytes(warps, --stages, chunkStride);
        if (smem > smemMax) return noalloc_fail(EP_ERR_INVALID, "row piece does not fit shared memory");
        // Raise (never lower) the kernel's dynamic shared-memory limit, so that
        // plans created with a larger limit keep working.
        int limit = 0;
        if ((e = ep::scatter_get_smem(&limit)) != cudaSuccess)
            return noalloc_fail(EP_ERR_CUDA, "cudaFuncGetAttributes: %s", cudaGetErrorString(e));
        if ((size_t)limit < smem && (e = ep::scatter_set_smem(smem)) != cudaSuccess)
            return noalloc_fail(EP_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        int perSm = 0;
        if ((e = ep::scatter_blocks_per_sm(warps, smem, &perSm)) != cudaSuccess || perSm < 1)
            return noalloc_fail(EP_ERR_CUDA, "occupancy query failed");

        ep::RouteParams rp{};
        rp.idx = topk_idx;
        rp.w = cfg->useWeights ? topk_w : nullptr;
        rp.route = route;
        rp.tok_mask = tok_mask;
        rp.tile_cnt = tile_cnt;
        rp.tile_base = tile_base;
        rp.recv_count = recv_count;
        rp.ticket = ticket;
        rp.work = work;
        rp.ptotal = ptotal;
        rp.lastScan = 1;  // the last block scans the tile counts
        rp.err = err;
        rp.G = (int)G;
        rp.W = W;
        rp.k = cfg->numExpertPerToken;
        rp.nEpr = cfg->numExpertPerRank;
        rp.E = W * cfg->numExpertPerRank;
        rp.numTiles = info.numTiles;
        rp.maxRecv = info.maxRecv;
        rp.useWeights = cfg->useWeights;
        if ((e = ep::launch_route_count(rp, false, s)) != cudaSuccess)
            return noalloc_fail(EP_ERR_CUDA, "launch route_count: %s", cudaGetErrorString(e));

        ep::ScatterParams sp{};
        sp.x = static_cast<const uint8_t*>(x);
        sp.idx = topk_idx;
        sp.route = route;
        sp.tok_mask = tok_mask;
        sp.tile_base = tile_base;
        sp.work = work;
        sp.ptotal = ptotal;
        sp.recv_x = static_cast<uint8_t*>(recv_x);
        sp.recv_meta = recv_meta;
        sp.err = err;
        sp.rowBytes = info.rowBytes;
        sp.G = (int)G;
        sp.W = W;
        sp.k = cfg->numExpertPerToken;
        sp.nEpr = cfg->numExpertPerRank;
        sp.E = W * cfg->numExpertPerRank;
        sp.T = cfg->maxTokPerRank;
        sp.maxRecv = info.maxRecv;
        sp.M = info.metaFields;
        sp.chunkBytes = info.scatterChunkBytes;
        sp.chunkStride = chunkStride;
        sp.numChunks = (int)((sp.rowBytes + sp.chunkBytes - 1) / sp.chunkBytes);
        sp.stages = stages;
        sp.baseShift = 8;  // route_count's 256-token tiles
        sp.baseStride = W + 1;
        sp.boundsRows = info.maxRecv;
        if ((e = ep::launch_scatter_rows(sp, false, ds.numSMs * perSm, warps, smem, s)) != cudaSuccess)
            return noalloc_fail(EP_ERR_CUDA, "launch scatter_rows: %s", cudaGetErrorString(e));
        return EP_OK;
    } catch (...) {
        return noalloc_fail(EP_ERR_INVALID, "unexpected exception");
    }
}
