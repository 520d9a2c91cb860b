// ep_internal.h -- parameter blocks and launchers shared by the C ABI layer
// (ep_abi.cu) and the kernels (ep_kernels.cu). Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ep {

// Tokens per routing tile: one 256-thread block counts one tile, one thread
// per token (flattened token index g = r*T + t, so tiles follow the
// (source rank, token) order that the slots follow).
constexpr int kCountTile = 256;
constexpr int kCountWarps = kCountTile / 32;
constexpr int kMaxWorld = 32;   // one destination bit per lane of a 32-bit mask
constexpr int kMaxTopk = 32;    // one topk entry per lane
constexpr int kMaxScatterWarps = 16;
constexpr int kMaxCombineWarps = 16;
// Bounded waits give up after this many SM clock cycles (about 1 s at 1.9 GHz).
constexpr long long kWaitCycles = 2000000000LL;

struct RouteParams {
    const int32_t* idx;     // [G][k]
    const float* w;         // [G][k] or nullptr (useWeights == 0)
    int2* route;            // [G][W]: (tile-local rank or -1, weight-sum bits)
    int32_t* tile_cnt;      // [numTiles][W]
    int32_t* tile_base;     // [numTiles][W], written by the last block
    int32_t* recv_count;    // [W]
    uint32_t* ticket;       // blocks finished this call; the last block resets it
    int32_t* err;           // device error word
    int G, W, k, nEpr, E, numTiles, maxRecv, useWeights;
};

struct ScatterParams {
    const uint8_t* x;          // [G][rowBytes]
    const int32_t* idx;        // [G][k]
    int2* route;               // [G][W]: in: tile-local rank; out: slot
    const int32_t* tile_base;  // [numTiles][W]
    uint8_t* recv_x;           // [W][maxRecv][rowBytes]
    int32_t* recv_meta;        // [W][maxRecv][M]
    int32_t* err;
    long long rowBytes;
    int G, W, k, nEpr, E, T, maxRecv, M;
    int chunkBytes;   // bytes per staged copy, multiple of 16
    int chunkStride;  // shared-memory bytes per stage, multiple of 128
    int numChunks;    // ceil(rowBytes / chunkBytes)
    int stages;       // stages per copy engine (>= 2)
};

struct CombineParams {
    const uint8_t* y;      // [W][maxRecv][rowBytes]
    const int2* route;     // [G][W]: (slot or -1, weight bits)
    uint8_t* out;          // [G][rowBytes]
    long long rowBytes;
    int G, W, maxRecv;
};

// Launchers (ep_kernels.cu). Each returns the cudaError_t of its launch.
cudaError_t launch_route_count(const RouteParams& p, cudaStream_t s);
// Scatter variants: TMA bulk copies staged in shared memory (kPend = bulk
// store groups left draining when a stage is refilled), or plain 16-byte
// register copies (no shared memory).
constexpr int kScatterTma = 0;
constexpr int kScatterRegs = 1;
cudaError_t launch_scatter_rows(const ScatterParams& p, int mode, int pend, int blocks, int warps,
                                size_t smem, cudaStream_t s);
cudaError_t launch_combine(const CombineParams& p, int blocks, int warps, cudaStream_t s);

// Shared-memory bytes the scatter kernel needs for a geometry.
size_t scatter_smem_bytes(int warps, int stages, int chunkStride);
// Opt the TMA scatter kernel in to `bytes` of dynamic shared memory.
cudaError_t scatter_set_smem(int pend, size_t bytes);
// Blocks of each kernel that fit on one SM (occupancy calculator).
cudaError_t scatter_blocks_per_sm(int mode, int pend, int warps, size_t smem, int* out);
cudaError_t combine_blocks_per_sm(int warps, int* out);
// Current dynamic shared-memory limit of the TMA scatter kernel.
cudaError_t scatter_get_smem(int pend, int* bytes);
// Replace this thread's ep_last_error() text.
void set_last_error(const char* msg);

}  // namespace ep
