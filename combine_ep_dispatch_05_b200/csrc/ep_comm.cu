// ep_comm.cu -- include/ep_comm.h: expert parallelism across processes, one
// rank per process. Memory, connection (CUDA IPC), and the call sequences of
// dispatch and combine; the kernels are those of ep_kernels.cu (route_count,
// scatter_rows and combine with per-destination bases, plus the count
// exchange / barrier and the push).
//
// Each rank owns two device allocations:
//   shared  mapped by every rank: count table int32 [W][W], barrier flags
//           u32 [W], receive rows [maxRecv][rowBytes], meta records
//           [maxRecv][3 + k], landing rows [T * min(W, k)][combine row];
//   local   the routing scratch of a plan over T tokens (ep_internal.h's
//           scratch layout), then this rank's count row, received-row count,
//           barrier epoch and the PeerTable the kernels read.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "ep.h"
#include "ep_comm.h"
#include "ep_internal.h"

namespace ep {
// Whether the combine reads y in 32-byte loads (ep_abi.cu): outputs of at
// least 192 MiB with rows a multiple of 32 bytes, unless EP_COMBINE_WIDE says.
bool combine_wide_loads(long long outBytes, long long rowBytes);
}

namespace {

constexpr char kMagic[8] = {'E', 'P', 'C', 'O', 'M', 'M', '1', '\0'};

// The connection record of a rank (EP_COMM_HANDLE_BYTES bytes).
struct Record {
    char magic[8];
    int32_t rank;
    int32_t sync;
    EpCfg cfg;
    uint64_t sharedBytes;
    unsigned char uuid[16];  // the rank's GPU
    cudaIpcMemHandle_t ipc;  // its shared allocation
};
static_assert(sizeof(Record) <= EP_COMM_HANDLE_BYTES, "connection record too large");

size_t up256(size_t n) { return (n + 255) & ~(size_t)255; }

int cuda_err(cudaError_t e, const char* what) {
    char msg[512];
    std::snprintf(msg, sizeof msg, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
    return ep::fail_code(e == cudaErrorMemoryAllocation ? EP_ERR_NOMEM : EP_ERR_CUDA, msg);
}

int err(int code, const char* msg) { return ep::fail_code(code, msg); }

bool aligned(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

}  // namespace

struct EpComm {
    EpCfg cfg;
    int rank, W, T, sync, device;
    EpHostBarrier barrier;
    void* ctx;
    ep::CopyGeometry geo;
    bool dense;
    int numTiles, maxRecv, M, maxLanding;
    long long rowBytes, crow;
    unsigned char uuid[16];
    unsigned slack;
    // shared allocation and its regions
    unsigned char* shared;
    size_t sharedBytes, offCounts, offFlags, offRecvX, offMeta, offLanding;
    // local allocation and its regions
    unsigned char* local;
    size_t localBytes;
    ep::ScratchLayout L;
    size_t offMyCount, offRecvTotal, offEpoch, offPeers;
    void* opened[ep::kMaxWorld];  // other ranks' shared allocations, mapped here
    bool connected, dispatched;
};

namespace {

void free_comm(EpComm* c) {
    if (!c) return;
    for (int q = 0; q < ep::kMaxWorld; ++q)
        if (c->opened[q]) cudaIpcCloseMemHandle(c->opened[q]);
    if (c->shared) cudaFree(c->shared);
    if (c->local) cudaFree(c->local);
    delete c;
}

// Host barrier of EP_SYNC_HOST: this rank's work so far is complete, then
// every rank meets.
int host_barrier(EpComm* c, cudaStream_t s, const char* where) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_err(e, "cudaStreamSynchronize");
    if (c->barrier(c->ctx) != 0) {
        char msg[256];
        std::snprintf(msg, sizeof msg, "rank %d: another rank did not arrive at the barrier %s", c->rank, where);
        return err(EP_ERR_PEER, msg);
    }
    return EP_OK;
}

ep::SyncParams sync_params(const EpComm* c, bool exchange) {
    ep::SyncParams p{};
    p.peers = reinterpret_cast<const ep::PeerTable*>(c->local + c->offPeers);
    p.myCount = reinterpret_cast<const int32_t*>(c->local + c->offMyCount);
    p.epoch = reinterpret_cast<unsigned*>(c->local + c->offEpoch);
    p.err = reinterpret_cast<int32_t*>(c->local + c->L.err);
    p.rank = c->rank;
    p.W = c->W;
    p.exchange = exchange ? 1 : 0;
    p.barrier = c->sync == EP_SYNC_DEVICE ? 1 : 0;
    p.slack = c->slack;
    return p;
}

int check_device(const EpComm* c) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_err(e, "cudaGetDevice");
    if (dev != c->device) return err(EP_ERR_DEVICE, "the current device is not the communicator's device");
    return EP_OK;
}

}  // namespace

extern "C" {

EpComm* ep_comm_create(const EpCfg* cfg, int32_t rank, int32_t sync, EpHostBarrier barrier, void* ctx) {
    EpComm* c = nullptr;
    try {
        if (ep::cfg_valid(cfg) != EP_OK) return nullptr;
        if (rank < 0 || rank >= cfg->worldSize) {
            err(EP_ERR_INVALID, "rank outside 0..worldSize-1");
            return nullptr;
        }
        if (sync != EP_SYNC_DEVICE && sync != EP_SYNC_HOST) {
            err(EP_ERR_INVALID, "sync must be EP_SYNC_DEVICE or EP_SYNC_HOST");
            return nullptr;
        }
        if (sync == EP_SYNC_HOST && !barrier) {
            err(EP_ERR_INVALID, "EP_SYNC_HOST needs a barrier function");
            return nullptr;
        }
        c = new (std::nothrow) EpComm();
        if (!c) {
            err(EP_ERR_NOMEM, "host allocation failed");
            return nullptr;
        }
        c->cfg = *cfg;
        c->rank = rank;
        c->W = cfg->worldSize;
        c->T = cfg->maxTokPerRank;
        c->sync = sync;
        c->barrier = barrier;
        c->ctx = ctx;
        if (ep::copy_geometry(cfg, &c->geo) != EP_OK) {
            free_comm(c);
            return nullptr;
        }
        c->device = c->geo.device;
        cudaDeviceProp prop;
        cudaError_t e = cudaGetDeviceProperties(&prop, c->device);
        if (e != cudaSuccess) {
            cuda_err(e, "cudaGetDeviceProperties");
            free_comm(c);
            return nullptr;
        }
        std::memcpy(c->uuid, prop.uuid.bytes, sizeof c->uuid);
        // Large batches take route_count's large-batch form (as plans do).
        c->dense = c->T > 16384;
        c->numTiles = (c->T + ep::kCountTile - 1) / ep::kCountTile;
        c->maxRecv = cfg->maxRecv == 0 ? c->W * c->T : cfg->maxRecv;
        c->M = 3 + cfg->numExpertPerToken;
        c->maxLanding = c->T * std::min(c->W, cfg->numExpertPerToken);
        const int es = cfg->dtype == EP_FP32 ? 4 : cfg->dtype == EP_BF16 ? 2 : 1;
        c->rowBytes = (long long)cfg->hiddenDim * es;
        const long long hc = cfg->dtype == EP_FP4X2 ? 2LL * cfg->hiddenDim : cfg->hiddenDim;
        c->crow = hc * (cfg->dtype == EP_FP32 ? 4 : 2);
        if (const char* t = std::getenv("EP_TEST_UNREACHABLE_BARRIER")) c->slack = std::strcmp(t, "1") == 0;

        c->offCounts = 0;
        c->offFlags = c->offCounts + up256(sizeof(int32_t) * c->W * c->W);
        c->offRecvX = c->offFlags + up256(sizeof(unsigned) * c->W);
        c->offMeta = c->offRecvX + up256((size_t)c->maxRecv * c->rowBytes);
        c->offLanding = c->offMeta + up256((size_t)c->maxRecv * c->M * sizeof(int32_t));
        c->sharedBytes = c->offLanding + up256((size_t)c->maxLanding * c->crow);

        c->L = ep::scratch_layout(c->T, c->W, c->numTiles);
        c->offMyCount = c->L.total;
        c->offRecvTotal = c->offMyCount + up256(sizeof(int32_t) * c->W);
        c->offEpoch = c->offRecvTotal + 256;
        c->offPeers = c->offEpoch + 256;
        c->localBytes = c->offPeers + up256(sizeof(ep::PeerTable));

        void* p = nullptr;
        if ((e = cudaMalloc(&p, c->sharedBytes)) != cudaSuccess) {
            cuda_err(e, "cudaMalloc(shared)");
            free_comm(c);
            return nullptr;
        }
        c->shared = static_cast<unsigned char*>(p);
        if ((e = cudaMalloc(&p, c->localBytes)) != cudaSuccess) {
            cuda_err(e, "cudaMalloc(local)");
            free_comm(c);
            return nullptr;
        }
        c->local = static_cast<unsigned char*>(p);
        if ((e = cudaMemset(c->shared, 0, c->sharedBytes)) != cudaSuccess ||
            (e = cudaMemset(c->local, 0, c->localBytes)) != cudaSuccess ||
            (e = cudaDeviceSynchronize()) != cudaSuccess) {
            cuda_err(e, "cudaMemset");
            free_comm(c);
            return nullptr;
        }
        ep::set_last_error("");
        return c;
    } catch (...) {
        err(EP_ERR_INVALID, "unexpected exception");
        free_comm(c);
        return nullptr;
    }
}

int ep_comm_handle(const EpComm* c, void* out) {
    try {
        if (!c || !out) return err(EP_ERR_INVALID, "comm or out is NULL");
        Record r;
        std::memset(&r, 0, sizeof r);
        std::memcpy(r.magic, kMagic, sizeof kMagic);
        r.rank = c->rank;
        r.sync = c->sync;
        r.cfg = c->cfg;
        r.sharedBytes = c->sharedBytes;
        std::memcpy(r.uuid, c->uuid, sizeof r.uuid);
        const cudaError_t e = cudaIpcGetMemHandle(&r.ipc, c->shared);
        if (e != cudaSuccess) return cuda_err(e, "cudaIpcGetMemHandle");
        std::memset(out, 0, EP_COMM_HANDLE_BYTES);
        std::memcpy(out, &r, sizeof r);
        return EP_OK;
    } catch (...) {
        return err(EP_ERR_INVALID, "unexpected exception");
    }
}

int ep_comm_connect(EpComm* c, const void* records) {
    try {
        if (!c || !records) return err(EP_ERR_INVALID, "comm or records is NULL");
        if (c->connected) return err(EP_ERR_STATE, "already connected");
        int rc = check_device(c);
        if (rc) return rc;
        const unsigned char* base = static_cast<const unsigned char*>(records);
        Record rec[ep::kMaxWorld];
        for (int q = 0; q < c->W; ++q) {
            std::memcpy(&rec[q], base + (size_t)q * EP_COMM_HANDLE_BYTES, sizeof(Record));
            if (std::memcmp(rec[q].magic, kMagic, sizeof kMagic) != 0)
                return err(EP_ERR_INVALID, "a connection record is not one of ep_comm_handle");
            if (rec[q].rank != q) return err(EP_ERR_INVALID, "connection records are not in rank order");
            if (std::memcmp(&rec[q].cfg, &c->cfg, sizeof(EpCfg)) != 0 || rec[q].sync != c->sync ||
                rec[q].sharedBytes != c->sharedBytes)
                return err(EP_ERR_INVALID, "the ranks' configurations differ");
        }
        if (c->sync == EP_SYNC_DEVICE)
            for (int a = 0; a < c->W; ++a)
                for (int b = a + 1; b < c->W; ++b)
                    if (std::memcmp(rec[a].uuid, rec[b].uuid, sizeof rec[a].uuid) == 0)
                        return err(EP_ERR_UNSUPPORTED,
                                   "EP_SYNC_DEVICE needs a GPU for every rank (two ranks share one); "
                                   "use EP_SYNC_HOST");
        ep::PeerTable t;
        std::memset(&t, 0, sizeof t);
        for (int q = 0; q < c->W; ++q) {
            unsigned char* sh = c->shared;
            if (q != c->rank) {
                void* p = nullptr;
                const cudaError_t e = cudaIpcOpenMemHandle(&p, rec[q].ipc, cudaIpcMemLazyEnablePeerAccess);
                if (e != cudaSuccess) {
                    for (int u = 0; u < q; ++u)
                        if (c->opened[u]) {
                            cudaIpcCloseMemHandle(c->opened[u]);
                            c->opened[u] = nullptr;
                        }
                    return cuda_err(e, "cudaIpcOpenMemHandle");
                }
                c->opened[q] = p;
                sh = static_cast<unsigned char*>(p);
            }
            t.recv_x[q] = sh + c->offRecvX;
            t.recv_meta[q] = reinterpret_cast<int32_t*>(sh + c->offMeta);
            t.landing[q] = sh + c->offLanding;
            t.counts[q] = reinterpret_cast<int32_t*>(sh + c->offCounts);
            t.flags[q] = reinterpret_cast<unsigned*>(sh + c->offFlags);
        }
        const cudaError_t e = cudaMemcpy(c->local + c->offPeers, &t, sizeof t, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_err(e, "cudaMemcpy(peer table)");
        c->connected = true;
        ep::set_last_error("");
        return EP_OK;
    } catch (...) {
        return err(EP_ERR_INVALID, "unexpected exception");
    }
}

int ep_comm_info(const EpComm* c, EpCommInfo* info) {
    if (!c || !info) return err(EP_ERR_INVALID, "comm or info is NULL");
    std::memset(info, 0, sizeof *info);
    info->rank = c->rank;
    info->worldSize = c->W;
    info->sync = c->sync;
    info->maxRecv = c->maxRecv;
    info->metaFields = c->M;
    info->maxLanding = c->maxLanding;
    info->rowBytes = c->rowBytes;
    info->combineRowBytes = c->crow;
    info->recvX = c->shared + c->offRecvX;
    info->recvMeta = reinterpret_cast<int32_t*>(c->shared + c->offMeta);
    info->recvCount = reinterpret_cast<int32_t*>(c->local + c->offRecvTotal);
    info->sharedBytes = (int64_t)c->sharedBytes;
    info->localBytes = (int64_t)c->localBytes;
    info->scatterBlocks = c->geo.blocks;
    info->scatterWarps = c->geo.warps;
    info->scatterStages = c->geo.stages;
    info->combineBlocks = c->geo.combineBlocks;
    info->combineWarps = c->geo.combineWarps;
    info->device = c->device;
    return EP_OK;
}

int ep_comm_dispatch(EpComm* c, const void* x, const int32_t* topk_idx, const float* topk_w, void* stream) {
    try {
        if (!c) return err(EP_ERR_INVALID, "comm is NULL");
        if (!c->connected) return err(EP_ERR_STATE, "ep_comm_connect has not run");
        if (!x || !topk_idx) return err(EP_ERR_INVALID, "x or topk_idx is NULL");
        if (c->cfg.useWeights && !topk_w) return err(EP_ERR_INVALID, "topk_w is NULL but useWeights is 1");
        if (!aligned(x, 16)) return err(EP_ERR_ALIGN, "x must be 16-byte aligned");
        if (!aligned(topk_idx, 4) || (topk_w && !aligned(topk_w, 4)))
            return err(EP_ERR_ALIGN, "topk_idx and topk_w must be 4-byte aligned");
        int rc = check_device(c);
        if (rc) return rc;
        cudaStream_t s = static_cast<cudaStream_t>(stream);
        const bool host = c->sync == EP_SYNC_HOST;
        // Every rank is here before any kernel of this call touches another rank.
        if (host && (rc = host_barrier(c, s, "at the start of dispatch")) != EP_OK) return rc;

        unsigned char* lb = c->local;
        int32_t* myCount = reinterpret_cast<int32_t*>(lb + c->offMyCount);
        ep::RouteParams rp{};
        rp.idx = topk_idx;
        rp.w = c->cfg.useWeights ? topk_w : nullptr;
        rp.route = reinterpret_cast<int2*>(lb + c->L.route);
        rp.tok_mask = reinterpret_cast<uint32_t*>(lb + c->L.tok_mask);
        rp.tile_cnt = reinterpret_cast<int32_t*>(lb + c->L.tile_cnt);
        rp.tile_base = reinterpret_cast<int32_t*>(lb + c->L.tile_base);
        rp.recv_count = myCount;  // the last block's column totals: this rank's count row
        rp.ticket = reinterpret_cast<uint32_t*>(lb + c->L.ticket);
        rp.work = reinterpret_cast<int32_t*>(lb + c->L.work);
        rp.ptotal = reinterpret_cast<int32_t*>(lb + c->L.ptotal);
        rp.err = reinterpret_cast<int32_t*>(lb + c->L.err);
        rp.G = c->T;
        rp.W = c->W;
        rp.k = c->cfg.numExpertPerToken;
        rp.nEpr = c->cfg.numExpertPerRank;
        rp.E = c->W * c->cfg.numExpertPerRank;
        rp.numTiles = c->numTiles;
        rp.maxRecv = c->maxRecv;
        rp.useWeights = c->cfg.useWeights;
        rp.lastScan = 1;
        cudaError_t e = ep::launch_route_count(rp, c->dense, s);
        if (e != cudaSuccess) return cuda_err(e, "launch route_count");

        // The count exchange (and, EP_SYNC_DEVICE, the barrier after it).
        if ((e = ep::launch_comm_sync(sync_params(c, true), s)) != cudaSuccess)
            return cuda_err(e, "launch count exchange");
        if (host && (rc = host_barrier(c, s, "after the count exchange")) != EP_OK) return rc;

        ep::ScatterParams sp{};
        sp.x = static_cast<const uint8_t*>(x);
        sp.idx = topk_idx;
        sp.route = rp.route;
        sp.tok_mask = rp.tok_mask;
        sp.tile_base = rp.tile_base;
        sp.work = rp.work;
        sp.ptotal = c->dense ? nullptr : rp.ptotal;
        sp.err = rp.err;
        sp.rowBytes = c->rowBytes;
        sp.G = c->T;
        sp.W = c->W;
        sp.k = c->cfg.numExpertPerToken;
        sp.nEpr = c->cfg.numExpertPerRank;
        sp.E = rp.E;
        sp.T = c->T;
        sp.maxRecv = c->maxRecv;
        sp.M = c->M;
        sp.chunkBytes = c->geo.chunkBytes;
        sp.chunkStride = c->geo.chunkStride;
        sp.numChunks = c->geo.numChunks;
        sp.stages = c->geo.stages;
        sp.baseShift = 8;
        sp.baseStride = c->dense ? c->W : c->W + 1;
        sp.numTiles = c->numTiles;
        sp.recv_count = myCount;
        sp.fanoutSwitch = 375;
        sp.peers = reinterpret_cast<const ep::PeerTable*>(lb + c->offPeers);
        sp.rank = c->rank;
        sp.counts = reinterpret_cast<const int32_t*>(c->shared + c->offCounts);
        sp.recv_total = reinterpret_cast<int32_t*>(lb + c->offRecvTotal);
        sp.boundsRows = c->maxRecv;
        e = ep::launch_scatter_rows(sp, c->dense, c->geo.blocks, c->geo.warps, c->geo.smem, s);
        if (e != cudaSuccess) return cuda_err(e, "launch scatter_rows");

        // Every rank's rows have arrived before anything reads them.
        if (host) {
            if ((rc = host_barrier(c, s, "after the scatter")) != EP_OK) return rc;
        } else if ((e = ep::launch_comm_sync(sync_params(c, false), s)) != cudaSuccess) {
            return cuda_err(e, "launch barrier");
        }
        c->dispatched = true;
        return EP_OK;
    } catch (...) {
        return err(EP_ERR_INVALID, "unexpected exception");
    }
}

int ep_comm_combine(EpComm* c, const void* y, void* out, void* stream) {
    try {
        if (!c) return err(EP_ERR_INVALID, "comm is NULL");
        if (!y || !out) return err(EP_ERR_INVALID, "y or out is NULL");
        if (!aligned(y, 16) || !aligned(out, 16)) return err(EP_ERR_ALIGN, "y and out must be 16-byte aligned");
        if (!c->dispatched) return err(EP_ERR_STATE, "combine before any dispatch");
        int rc = check_device(c);
        if (rc) return rc;
        cudaStream_t s = static_cast<cudaStream_t>(stream);
        const bool host = c->sync == EP_SYNC_HOST;
        if (host && (rc = host_barrier(c, s, "at the start of combine")) != EP_OK) return rc;

        ep::PushParams pp{};
        pp.y = static_cast<const uint8_t*>(y);
        pp.peers = reinterpret_cast<const ep::PeerTable*>(c->local + c->offPeers);
        pp.counts = reinterpret_cast<const int32_t*>(c->shared + c->offCounts);
        pp.err = reinterpret_cast<int32_t*>(c->local + c->L.err);
        pp.rowBytes = c->crow;
        pp.rank = c->rank;
        pp.W = c->W;
        pp.maxRecv = c->maxRecv;
        pp.maxLanding = c->maxLanding;
        cudaError_t e = ep::launch_comm_push(pp, c->geo.numSMs * 4, s);
        if (e != cudaSuccess) return cuda_err(e, "launch push");

        // Every rank's expert outputs have landed before any rank folds them.
        if (host) {
            if ((rc = host_barrier(c, s, "after the push")) != EP_OK) return rc;
        } else if ((e = ep::launch_comm_sync(sync_params(c, false), s)) != cudaSuccess) {
            return cuda_err(e, "launch barrier");
        }

        ep::CombineParams cp{};
        cp.y = c->shared + c->offLanding;
        cp.route = reinterpret_cast<const int2*>(c->local + c->L.route);
        cp.out = static_cast<uint8_t*>(out);
        cp.work = reinterpret_cast<int32_t*>(c->local + c->L.cwork);
        cp.done = reinterpret_cast<uint32_t*>(c->local + c->L.cdone);
        cp.rowBytes = c->crow;
        cp.G = c->T;
        cp.W = c->W;
        cp.maxRecv = c->maxRecv;
        cp.counts = reinterpret_cast<const int32_t*>(c->shared + c->offCounts);
        cp.rank = c->rank;
        cp.err = pp.err;
        cp.yBytes = (long long)c->maxLanding * c->crow;
        // 32-byte loads by the one-GPU plans' rule on this rank's output (its T
        // tokens); the landing rows start 256-byte aligned, crow apart.
        const bool wide = ep::combine_wide_loads((long long)c->T * c->crow, c->crow) &&
                          reinterpret_cast<uintptr_t>(cp.y) % 32 == 0;
        e = ep::launch_combine(cp, c->cfg.dtype == EP_FP32, wide, c->geo.combineBlocks, c->geo.combineWarps, s);
        if (e != cudaSuccess) return cuda_err(e, "launch combine");
        return EP_OK;
    } catch (...) {
        return err(EP_ERR_INVALID, "unexpected exception");
    }
}

int ep_comm_check_error(EpComm* c) {
    if (!c) return err(EP_ERR_INVALID, "comm is NULL");
    int rc = check_device(c);
    if (rc) return rc;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_err(e, "cudaDeviceSynchronize");
    int32_t word = 0;
    int32_t* w = reinterpret_cast<int32_t*>(c->local + c->L.err);
    if ((e = cudaMemcpy(&word, w, sizeof word, cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_err(e, "cudaMemcpy(error word)");
    if ((e = cudaMemset(w, 0, sizeof word)) != cudaSuccess) return cuda_err(e, "cudaMemset");
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_err(e, "cudaDeviceSynchronize");
    return word;
}

void ep_comm_destroy(EpComm* c) { free_comm(c); }

int ep_comm_barrier_selftest(int32_t W, int32_t rounds, int32_t absentRank, int32_t absentFrom,
                             int32_t* roundsDone, int32_t* errors, int32_t* violations) {
    try {
        if (W < 1 || W > ep::kMaxWorld) return err(EP_ERR_INVALID, "W outside 1..32");
        if (rounds < 1 || rounds > 100000) return err(EP_ERR_INVALID, "rounds outside 1..100000");
        const size_t flagsOff = up256(sizeof(ep::PeerTable));
        const size_t epochsOff = flagsOff + up256(sizeof(unsigned) * W * W);
        const size_t errsOff = epochsOff + up256(sizeof(unsigned) * W);
        const size_t dataOff = errsOff + up256(sizeof(int32_t) * W);
        const size_t doneOff = dataOff + up256(sizeof(int32_t) * (size_t)W * rounds);
        const size_t violOff = doneOff + up256(sizeof(int32_t) * W);
        const size_t total = violOff + up256(sizeof(int32_t) * W);
        unsigned char* mem = nullptr;
        cudaError_t e = cudaMalloc(reinterpret_cast<void**>(&mem), total);
        if (e != cudaSuccess) return cuda_err(e, "cudaMalloc");
        ep::PeerTable t;
        std::memset(&t, 0, sizeof t);
        for (int r = 0; r < W; ++r) t.flags[r] = reinterpret_cast<unsigned*>(mem + flagsOff) + (size_t)r * W;
        ep::BarrierTestParams p{};
        p.peers = reinterpret_cast<ep::PeerTable*>(mem);
        p.epochs = reinterpret_cast<unsigned*>(mem + epochsOff);
        p.errs = reinterpret_cast<int32_t*>(mem + errsOff);
        p.data = reinterpret_cast<int32_t*>(mem + dataOff);
        p.rounds_done = reinterpret_cast<int32_t*>(mem + doneOff);
        p.violations = reinterpret_cast<int32_t*>(mem + violOff);
        p.W = W;
        p.rounds = rounds;
        p.absent = absentRank;
        p.absentFrom = absentFrom;
        int32_t out[3][ep::kMaxWorld];
        if ((e = cudaMemset(mem, 0, total)) != cudaSuccess ||
            (e = cudaMemcpy(mem, &t, sizeof t, cudaMemcpyHostToDevice)) != cudaSuccess ||
            (e = ep::launch_comm_barrier_test(p, nullptr)) != cudaSuccess || (e = cudaDeviceSynchronize()) != cudaSuccess ||
            (e = cudaMemcpy(out[0], p.rounds_done, sizeof(int32_t) * W, cudaMemcpyDeviceToHost)) != cudaSuccess ||
            (e = cudaMemcpy(out[1], p.errs, sizeof(int32_t) * W, cudaMemcpyDeviceToHost)) != cudaSuccess ||
            (e = cudaMemcpy(out[2], p.violations, sizeof(int32_t) * W, cudaMemcpyDeviceToHost)) != cudaSuccess) {
            cudaFree(mem);
            return cuda_err(e, "barrier self-test");
        }
        cudaFree(mem);
        for (int r = 0; r < W; ++r) {
            if (roundsDone) roundsDone[r] = out[0][r];
            if (errors) errors[r] = out[1][r];
            if (violations) violations[r] = out[2][r];
        }
        return EP_OK;
    } catch (...) {
        return err(EP_ERR_INVALID, "unexpected exception");
    }
}

}  // extern "C"
