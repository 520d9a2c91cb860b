// ep_internal.h -- parameter blocks and launchers shared by the C ABI layer
// (ep_abi.cu) and the kernels (ep_kernels.cu). Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ep.h"

namespace ep {

// Tokens per routing tile: one 256-thread block counts one tile, one thread
// per token (flattened token index g = r*T + t, so tiles follow the
// (source rank, token) order that the slots follow).
constexpr int kCountTile = 256;
constexpr int kCountWarps = kCountTile / 32;
constexpr int kMaxWorld = 32;   // one destination bit per lane of a 32-bit mask
constexpr int kMaxTopk = 32;    // one topk entry per lane
constexpr int kMaxScatterWarps = 16;
constexpr int kMaxCombineWarps = 8;
// Warps of a dispatch_fused block (its first warps are the copy engines), and
// the most tokens one block may own (the plan takes dispatch_fused only when
// ceil(G / blocks) is at most this).
constexpr int kFusedWarps = 8;
constexpr int kFusedMaxOwn = 64;
// Shared memory kept back from the dynamic budget for the kernels' static
// shared memory.
constexpr size_t kStaticSmemReserve = 2048;
// The bounds-checking build (-DEP_DEBUG_BOUNDS, libep_b200_debug.so) checks
// every row, record and scale-row address of the copies against its buffer's
// extent; an access outside it is skipped and EP_DEVERR_BOUNDS is set.
#ifdef EP_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif
// Bounded waits give up after this many SM clock cycles (about 1 s at 1.9 GHz).
constexpr long long kWaitCycles = 2000000000LL;

// Ranks in separate processes (one GPU each): where every rank's shared
// buffers are mapped in this process, and this rank's copy of the count
// table. Lives in device memory; the kernels read it through a pointer.
struct PeerTable {
    uint8_t* recv_x[kMaxWorld];     // rank q's receive rows [maxRecv][rowBytes]
    int32_t* recv_meta[kMaxWorld];  // rank q's meta records [maxRecv][M]
    uint8_t* landing[kMaxWorld];    // rank q's landing rows of the push combine [maxLanding][combine row]
    int32_t* counts[kMaxWorld];     // rank q's count table [W][W]: row r = rows source r sends to each rank
    unsigned* flags[kMaxWorld];     // rank q's barrier flags [W]: the last epoch each rank arrived at
};

struct RouteParams {
    const int32_t* idx;     // [G][k]
    const float* w;         // [G][k] or nullptr (useWeights == 0)
    int2* route;            // [G][W]: (tile-local rank or -1, weight-sum bits)
    uint32_t* tok_mask;     // [G]: destination mask of each token
    int32_t* tile_cnt;      // [numTiles][W + 1]: rows at each destination, present tokens
    int32_t* tile_base;     // [numTiles][W + 1], written by the last block (lastScan)
    int32_t* recv_count;    // [W], stored by the last block (lastScan)
    uint32_t* ticket;       // blocks finished this call; the last block resets it
    int32_t* work;          // scatter token counter; block 0 resets it
    int32_t* ptotal;        // present tokens of the call, stored by the last block (lastScan)
    int32_t* err;           // device error word
    int G, W, k, nEpr, E, numTiles, maxRecv, useWeights;
    int lastScan;           // 1: the last block scans the tile counts; 0: the scatter does
};

struct ScatterParams {
    const uint8_t* x;          // [G][rowBytes]
    const int32_t* idx;        // [G][k]
    int2* route;               // [G][W]: in: tile-local rank; out: slot
    const uint32_t* tok_mask;  // [G]: destination mask of each token
    const int32_t* tile_base;  // [numTiles][baseStride]: bases computed in global memory, or
    const int32_t* tile_cnt;   // [numTiles][W + 1]: route_count's counts, scanned by each block
    int baseStride;            // W + 1 (route_count tiles) or W (fused chunks)
    int baseSmemBytes;         // > 0: each block scans tile_cnt into this much shared memory
    int baseOffset;            // shared-memory byte offsets of the tile bases and of the engines
    int engineOffset;
    int numTiles;
    int32_t* work;             // next token to hand out (starts at 0 each call)
    const int32_t* ptotal;     // present tokens of the call (route_count's last block), or nullptr
    uint8_t* recv_x;           // [W][maxRecv][rowBytes]
    int32_t* recv_meta;        // [W][maxRecv][M]
    int32_t* err;
    long long rowBytes;
    int G, W, k, nEpr, E, T, maxRecv, M;
    int chunkBytes;   // bytes per staged copy, multiple of 16
    int chunkStride;  // shared-memory bytes per stage, multiple of 128
    int numChunks;    // ceil(rowBytes / chunkBytes)
    int stages;       // stages per copy engine (>= 2)
    int baseShift;    // tile_base has one row per 2^baseShift tokens (8: route_count tiles; 5: fused chunks)
    int fanoutSwitch;        // x100: above this mean fan-out (rows per token) one engine per block sits out (0: never)
    const uint32_t* scales;  // [G][scaleWords] per-token scale rows, or nullptr
    uint32_t* recv_scales;   // [W][maxRecv][scaleWords]
    int scaleWords;          // 0: no scale rows
    // Ranks in separate processes (nullptr: the W ranks are regions of recv_x /
    // recv_meta on this GPU). recv_count above is then this rank's count row.
    const PeerTable* peers;
    int rank;                // this rank (source of every token of the call)
    const int32_t* counts;   // this rank's count table [W][W], complete (after the exchange)
    int32_t* recv_total;     // rows this rank receives, stored by block 0
    int boundsRows;          // bounds-checking build: rows of each destination's buffers (maxRecv)
    int earlyIssue;          // row loads a copy engine issues before its ready hook: 0 all, n > 0 at most n, < 0 none
    // Only dispatch_fused uses these, and the fields below:
    const float* w;          // [G][k] or nullptr
    int32_t* recv_count;     // [W]
    int useWeights;
    unsigned barrierSlack;   // 0; 1 makes the look-back wait for a tag no block publishes (tests of the timeout path)
    int nEprShift;           // log2(nEpr) when nEpr is a power of two, else -1
    // (and engineOffset): the most tokens a block owns, its copy-engine warps,
    // the blocks' published totals [blocks][ceil(W / 6)], the call epoch and
    // the blocks past their look-back (the last one advances the epoch).
    int fusedOwn;
    int fusedEngines;
    unsigned long long* fused_agg;
    unsigned* fused_epoch;
    unsigned* fused_done;
};

// Byte offsets of dispatch_fused's routing area in shared memory (each
// 16-byte aligned): masks of the own chunks' tokens [chunks * 32], their own
// tokens per destination, then bases [chunks][W], the own tokens' slots
// [own][W], the present own tokens [own], counters ([0] present own tokens,
// [1] next one to hand out, [2 + pe] the block's total at pe), and the own
// tokens' topk ids and weights [own][k] each. own: the most tokens a block
// owns; its tokens span at most (own + 62) / 32 chunks.
struct FusedLayout {
    size_t cmask, ccnt, slot, list, ctr, ids, wts, total;
};
__host__ __device__ inline size_t fused_up16(size_t n) { return (n + 15) & ~(size_t)15; }
__host__ __device__ inline FusedLayout fused_layout(int own, int W, int warps, int k) {
    (void)warps;
    const size_t chunks = (size_t)(own + 62) / 32;
    FusedLayout L;
    L.cmask = 0;
    L.ccnt = L.cmask + fused_up16(chunks * 32 * 4);
    L.slot = L.ccnt + fused_up16(chunks * (size_t)W * 4);
    L.list = L.slot + fused_up16((size_t)own * W * 4);
    L.ctr = L.list + fused_up16((size_t)own * 4);
    L.ids = L.ctr + fused_up16((2 + kMaxWorld) * 4);
    L.wts = L.ids + fused_up16((size_t)own * k * 4);
    L.total = (L.wts + (size_t)own * k * 4 + 127) & ~(size_t)127;
    return L;
}

struct CombineParams {
    const uint8_t* y;      // [W][maxRecv][rowBytes]
    const int2* route;     // [G][W]: (slot or -1, weight bits)
    uint8_t* out;          // [G][rowBytes]
    int32_t* work;         // next token to hand out (0 at the start of each call)
    uint32_t* done;        // blocks finished; the last one resets work and done
    long long rowBytes;    // bytes of a y / out row (the combine leg's row)
    int G, W, maxRecv;
    // Ranks in separate processes: y is this rank's landing rows, where the
    // rows of destination pe start after those of the destinations before it
    // (counts: this rank's count table; nullptr: one GPU, y = [W][maxRecv]).
    const int32_t* counts;
    int rank;
    int32_t* err;          // the call is skipped when a barrier of it gave up (counts != nullptr)
    long long yBytes;      // bounds-checking build: bytes of y
};

// The count exchange and the barrier of ranks in separate processes (one
// block of 32 threads).
struct SyncParams {
    const PeerTable* peers;
    const int32_t* myCount;  // this rank's count row [W] (route_count's scan)
    unsigned* epoch;         // barriers this rank has passed (its own, on the device)
    int32_t* err;
    int rank, W;
    int exchange;            // 1: copy this rank's count row into row `rank` of every rank's count table
    int barrier;             // 1: then wait until every rank has arrived at this barrier
    unsigned slack;          // 0; test hook: 1 waits for an epoch that no rank reaches
};

// The push half of the combine of ranks in separate processes: every row
// this rank received goes back, as its expert output, to the landing rows
// of the rank it came from.
struct PushParams {
    const uint8_t* y;         // this rank's expert outputs [maxRecv][rowBytes]
    const PeerTable* peers;
    const int32_t* counts;    // this rank's count table [W][W]
    int32_t* err;
    long long rowBytes;       // bytes of a combine row
    int rank, W, maxRecv, maxLanding;
};

// Byte offsets of the dispatch scratch regions (each 256-byte aligned):
// routing table, token masks, tile counts, tile bases (256-token tiles of the
// split dispatch), the fused dispatch's published totals, the counters (one
// 256-byte region: tile ticket, scatter token counter, combine token counter,
// combine blocks done, route_count's present-token total, the fused
// dispatch's call epoch and blocks done), error word.
struct ScratchLayout {
    size_t route, tok_mask, tile_cnt, tile_base, fused_agg;
    size_t ticket, work, cwork, cdone, ptotal, fused_epoch, fused_done, err, total;
};

// fusedBlocks: the grid of dispatch_fused (0: the plan does not take it).
inline ScratchLayout scratch_layout(long long G, int W, int numTiles, int fusedBlocks = 0) {
    auto up = [](size_t n) { return (n + 255) & ~(size_t)255; };
    ScratchLayout L;
    L.route = 0;
    L.tok_mask = L.route + up(sizeof(int2) * (size_t)G * W);
    L.tile_cnt = L.tok_mask + up(sizeof(uint32_t) * (size_t)G);
    L.tile_base = L.tile_cnt + up(sizeof(int32_t) * (size_t)numTiles * (W + 1));
    L.fused_agg = L.tile_base + up(sizeof(int32_t) * (size_t)numTiles * (W + 1));
    L.ticket = L.fused_agg + up(sizeof(unsigned long long) * (size_t)fusedBlocks * ((W + 5) / 6));
    L.work = L.ticket + 4;
    L.cwork = L.ticket + 8;
    L.cdone = L.ticket + 12;
    L.ptotal = L.ticket + 16;
    L.fused_epoch = L.ticket + 20;
    L.fused_done = L.ticket + 24;
    L.err = L.ticket + 256;
    L.total = L.err + 256;
    return L;
}

// Launchers (ep_kernels.cu). Each returns the cudaError_t of its launch.
// dense: the large-batch form (tile counts at the W destinations only, last-block
// scan, tile bases with stride W); else W + 1 columns, lastScan as set.
cudaError_t launch_route_count(const RouteParams& p, bool dense, cudaStream_t s);
// The scatter: TMA bulk copies staged in shared memory. dense: the
// large-batch instance (shared hand-out, tile bases in global memory with
// stride W, no scan of its own).
cudaError_t launch_scatter_rows(const ScatterParams& p, bool dense, int blocks, int warps, size_t smem,
                                cudaStream_t s);
// fp32: float32 combine leg (an fp32 plan); bf16 otherwise. wide: 32-byte
// loads of y (y and rowBytes multiples of 32 bytes).
cudaError_t launch_combine(const CombineParams& p, bool fp32, bool wide, int blocks, int warps, cudaStream_t s);
// The fused dispatch of small batches: one launch, per-block routing
// (dispatch_fused, kFusedWarps warps per block): opt-in, occupancy, launch.
cudaError_t fused_set_smem(int W, int topk, size_t bytes);
cudaError_t fused_blocks_per_sm(int W, int topk, size_t smem, int* out);
cudaError_t launch_dispatch_fused(const ScatterParams& p, int blocks, size_t smem, cudaStream_t s);

// Ranks in separate processes: the count exchange / barrier, and the push.
cudaError_t launch_comm_sync(const SyncParams& p, cudaStream_t s);

// The barrier of EP_SYNC_DEVICE with W ranks emulated by the W blocks of one
// cooperative launch on this GPU (ep_comm_barrier_selftest).
struct BarrierTestParams {
    PeerTable* peers;      // flags[r] = rank r's flags [W]
    unsigned* epochs;      // [W] each emulated rank's epoch
    int32_t* errs;         // [W] each rank's error word
    int32_t* data;         // [W][rounds] what each rank wrote before each barrier
    int32_t* rounds_done;  // [W] barriers each rank completed
    int32_t* violations;   // [W] values a rank read after a barrier that were not yet written
    int W, rounds, absent, absentFrom;
};
cudaError_t launch_comm_barrier_test(const BarrierTestParams& p, cudaStream_t s);
cudaError_t launch_comm_push(const PushParams& p, int blocks, cudaStream_t s);

// Shared-memory bytes the scatter kernel needs for a geometry.
size_t scatter_smem_bytes(int warps, int stages, int chunkStride);
// Shared memory for the tile bases when the scatter scans route_count's tile
// counts itself ([numTiles][W + 1] ints, rounded up to 128 bytes).
size_t scatter_base_smem_bytes(int numTiles, int W);
constexpr size_t kMaxBaseSmemBytes = 16384;
// Opt a kernel in to `bytes` of dynamic shared memory (these only ever raise
// the limit, so that plans made earlier keep theirs).
cudaError_t scatter_set_smem(size_t bytes);
// Blocks of each kernel that fit on one SM (occupancy calculator).
cudaError_t scatter_blocks_per_sm(int warps, size_t smem, int* out);
cudaError_t combine_blocks_per_sm(int warps, bool fp32, int* out);
// Current dynamic shared-memory limit of the scatter kernel.
cudaError_t scatter_get_smem(int* bytes);
// Replace this thread's ep_last_error() text; fail_code also returns `code`.
void set_last_error(const char* msg);
int fail_code(int code, const char* msg);
// ep_cfg_check's rules, without clearing the last error first.
int cfg_valid(const EpCfg* cfg);

// Copy and combine geometry of a plan on the current device (route_count's
// last block scans the tile counts); EP_OK or a negative code.
struct CopyGeometry {
    int chunkBytes, chunkStride, numChunks;
    int warps, stages, blocks;  // copy engines per block, stages per engine, scatter grid
    size_t smem;                // the scatter's dynamic shared memory
    int combineWarps, combineBlocks;
    int numSMs, device;
};
int copy_geometry(const EpCfg* cfg, CopyGeometry* out);

}  // namespace ep
