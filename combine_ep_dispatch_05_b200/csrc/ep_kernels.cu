// ep_kernels.cu -- sm_100a kernels of MoE expert-parallel dispatch / combine
// over W virtual ranks held in one GPU's memory.
//
// dispatch = route_count (one launch) + scatter_rows (one launch)
//   route_count  one thread per token: destination mask (destPe = expert /
//                numExpertPerRank, "MORI JIT v2" design page §8), per-destination
//                weight sums, per-tile histogram by warp ballots, tile-local
//                ranks. For large batches the last block to finish scans the
//                tile histogram into per-(tile, destPe) bases and stores
//                recv_count (mori PR #599: a stored count); for small batches
//                every scatter block scans it in its own shared memory.
//                Slots end up ordered by (srcRank, token).
//   scatter_rows persistent copy engines, one per warp: each x row is read once
//                from HBM into shared memory by a TMA bulk copy
//                (cp.async.bulk, mbarrier completion) and written to every
//                destination by TMA bulk stores from the same shared memory,
//                while the warp's lanes write the meta records. The pages' copy
//                loops (WarpCopy on gfx9xx, one TDM tile per token on gfx1250,
//                design page §9 and PR #599) are the prior art.
// combine = combine (one launch)
//   combine      one warp per token: 4 destination rows x 4 16-byte columns
//                in flight per lane (read as 32-byte loads for large outputs),
//                float32 fma fold in destPe order; bf16 RNE out (float32 out,
//                unrounded, for a float32 plan).
// Option: dispatch_fused, the whole dispatch of a small batch in one launch
// (each block routes and copies its own share of the batch; the bases come
// from the other blocks' published counts by decoupled look-back).
//
// No kernel traps or spins without a bound: waits on shared-memory barriers
// and on other blocks' published words give up after kWaitCycles, set
// EP_DEVERR_TIMEOUT and drain their copies.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ep.h"
#include "ep_internal.h"

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// ------------------------------------------------------------- TMA / mbarrier
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of an mbarrier, giving up after kWaitCycles.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitCycles) return false;
    }
    return true;
}

// Global -> shared bulk copy; completion is counted on the mbarrier in bytes.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Shared -> global bulk copy, tracked by this thread's bulk async-groups.
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Every bulk group of this thread has completed (writes done).
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while the previous kernel of the stream finishes;
// pdl_wait() blocks until that kernel has completed and its writes are
// visible (a no-op without the launch attribute). pdl_trigger() lets the next
// kernel of the stream start its launch early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" :::); }

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 32 bytes (two 16-byte vectors) in one load; p must be 32-byte aligned.
__device__ __forceinline__ void ld_stream_v8(const void* p, uint4& a, uint4& b) {
    asm("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
        : "l"(p));
}

// =====================================================================
// Token hand-out shared by the scatter engines and the combine warps. Worker w
// of nU takes tokens w, w + nU, ... for R rounds (no coordination), then the
// rest, about the last eighth of the tokens, one at a time from a global
// counter, so that workers whose tokens had more destinations do not leave a
// tail (the spread of a worker's total over ~100 tokens is a few percent).
// With fewer than eight tokens per worker the split is static only: the
// counter would put thousands of atomics on one address for little balance.
// Workers are numbered warp-major (worker = warp * blocks + block), so that
// the static rounds give every block, i.e. every SM, the same number of
// tokens to within one per warp (block-major numbering gave the first blocks
// all the extra tokens: 15 against 12 per SM for 2048 tokens on 444 engines).
// =====================================================================
struct TokenSource {
    int w, nU, R, G, i;
    bool dyn;
    int32_t* ctr;
};

// P: the tokens that carry work (present tokens when the caller knows them,
// else G); the counter is used only when there are minPer of them per worker
// (8 for the scatter; the combine's 4: B200, main shape at 2048 tokens a
// rank, 235.4 us with the counter against 240.9 without).
__device__ __forceinline__ TokenSource make_source(int w, int nU, int G, int32_t* ctr, int P, int minPer = 8) {
    TokenSource s;
    s.w = w;
    s.nU = nU;
    s.G = G;
    s.i = 0;
    s.ctr = ctr;
    s.dyn = G >= minPer * nU && P >= minPer * nU;
    s.R = s.dyn ? max(0, (int)((7LL * G) / (8LL * nU)) - 1) : (G + nU - 1) / nU;
    return s;
}

// Next token of this worker, or G when it has none left.
__device__ __forceinline__ int source_next(TokenSource& s) {
    if (s.i < s.R) {
        const int t = s.w + (s.i++) * s.nU;
        if (t < s.G) return t;
        s.i = s.R;
    }
    if (!s.dyn) return s.G;
    const int t = s.R * s.nU + atomicAdd(s.ctr, 1);
    return t < s.G ? t : s.G;
}

// =====================================================================
// route_count: mask, weight sums, tile histogram, tile-local ranks; for large
// batches the last block scans the histogram, for small batches every
// scatter block does. kW = compile-time bound on W (8, 16 or 32).
// =====================================================================
// Destination mask and per-destination weight sums of token g (float32 fold
// in topk order); ids < 0 are masked, ids >= E are reported and masked. kK
// bounds k: all k ids and weights are loaded into registers first, so their
// loads are in flight together.
template <int kW, int kK>
__device__ __forceinline__ uint32_t route_token(const int32_t* idx, const float* w, int g, int k, int nEpr,
                                                int E, float (&ws)[kW], bool& bad) {
    uint32_t mask = 0;
#pragma unroll
    for (int pe = 0; pe < kW; ++pe) ws[pe] = 0.0f;
    const int32_t* ids = idx + (size_t)g * k;
    const float* wts = w ? w + (size_t)g * k : nullptr;
    int e_j[kK];
    float w_j[kK];
#pragma unroll
    for (int j = 0; j < kK; ++j) {
        e_j[j] = j < k ? ids[j] : -1;
        w_j[j] = (wts && j < k) ? wts[j] : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < kK; ++j) {
        const int e = e_j[j];
        if (e < 0) continue;  // masked entry (or j >= k)
        if (e >= E) {         // contract violation: report, treat as masked
            bad = true;
            continue;
        }
        const int pe_j = e / nEpr;
        mask |= 1u << pe_j;
        if (wts) {
#pragma unroll
            for (int pe = 0; pe < kW; ++pe)
                if (pe == pe_j) ws[pe] = ws[pe] + w_j[j];  // fold in topk order
        }
    }
    return mask;
}

// kDense: the form for large batches -- tile counts at the W destinations
// only, scanned by the last block, which also restarts the scatter's token
// counter. Otherwise the tile counts carry a column of present tokens (W + 1
// columns) and the scatter may scan them itself (lastScan == 0).
template <int kW, int kK, bool kDense>
__global__ void __launch_bounds__(kCountTile) ep_route_count_kernel(RouteParams p) {
    __shared__ int s_wcnt[kCountWarps][kW + 1];
    __shared__ int s_wpre[kCountWarps][kW];
    __shared__ int s_last;

    pdl_wait();     // the ids may come from the previous kernel of the stream
    pdl_trigger();  // let the scatter's launch and prologue overlap this kernel

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = blockIdx.x * kCountTile + tid;
    const int W = p.W, k = p.k, C = kDense ? W : W + 1;
    // The previous call's scatter has finished: its token counter restarts.
    if (!kDense && blockIdx.x == 0 && tid == 0) *p.work = 0;

    uint32_t mask = 0;
    bool bad = false;
    float ws[kW];
    if (g < p.G) mask = route_token<kW, kK>(p.idx, p.w, g, k, p.nEpr, p.E, ws, bad);
    if (bad) atomicOr(p.err, EP_DEVERR_EXPERT_RANGE);

    // Per-warp histogram by ballot; column W counts the present tokens.
#pragma unroll
    for (int pe = 0; pe < kW; ++pe) {
        if (pe < W) {
            const uint32_t b = __ballot_sync(kFull, (mask >> pe) & 1u);
            if (lane == 0) s_wcnt[warp][pe] = __popc(b);
        }
    }
    if (!kDense) {
        const uint32_t bp = __ballot_sync(kFull, mask != 0u);
        if (lane == 0) s_wcnt[warp][W] = __popc(bp);
    }
    __syncthreads();
    if (tid < C) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kCountWarps; ++w) {
            if (tid < W) s_wpre[w][tid] = run;
            run += s_wcnt[w][tid];
        }
        p.tile_cnt[blockIdx.x * C + tid] = run;
    }
    __syncthreads();

    if (g < p.G) p.tok_mask[g] = mask;

    // Tile-local rank of this token at each destination, and its weight sum.
    const uint32_t lt = lanemask_lt();
#pragma unroll
    for (int pe = 0; pe < kW; ++pe) {
        if (pe < W) {
            const bool hit = (mask >> pe) & 1u;
            const uint32_t b = __ballot_sync(kFull, hit);
            if (g < p.G) {
                int2 v;
                v.x = hit ? s_wpre[warp][pe] + __popc(b & lt) : -1;
                const float wsum = hit ? (p.useWeights ? ws[pe] : 1.0f) : 0.0f;
                v.y = __float_as_int(wsum);
                p.route[(size_t)g * W + pe] = v;
            }
        }
    }

    // When the scatter scans the tile counts itself, this block is done.
    if (!kDense && !p.lastScan) return;

    // Otherwise the last block to finish turns the tile histogram into
    // per-tile bases (column W: present tokens before the tile), stores
    // recv_count and the call's present-token total.
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(p.ticket, 1u) == (unsigned)(p.numTiles - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int pe = warp; pe < C; pe += kCountWarps) {
        int running = 0;
        for (int t0 = 0; t0 < p.numTiles; t0 += 32 * 8) {
            int v[8];  // 8 rows of 32 tiles: all loads in flight before the scans
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int t = t0 + 32 * u + lane;
                v[u] = t < p.numTiles ? __ldcg(p.tile_cnt + (size_t)t * C + pe) : 0;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int t = t0 + 32 * u + lane;
                int incl = v[u];
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int n = __shfl_up_sync(kFull, incl, off);
                    if (lane >= off) incl += n;
                }
                if (t < p.numTiles) p.tile_base[(size_t)t * C + pe] = running + incl - v[u];
                running += __shfl_sync(kFull, incl, 31);
            }
        }
        if (lane == 0) {
            if (pe < W) {
                p.recv_count[pe] = running;  // stored, not accumulated
                if (running > p.maxRecv) atomicOr(p.err, EP_DEVERR_CAPACITY);
            } else {
                *p.ptotal = running;
            }
        }
    }
    if (tid == 0) {  // ready for the scatter and for the next call (graph replay too)
        if (kDense) *p.work = 0;
        *p.ticket = 0u;
    }
}

// The scatter's own scan of route_count's tile counts ([numTiles][W + 1]),
// by one block into its shared memory: s_base[t][pe] = rows at pe of the
// tiles before t (column W: present tokens). Block 0 stores recv_count.
// Returns the call's present tokens; *rows = the rows of all destinations.
// Returns -1 (after setting EP_DEVERR_TIMEOUT) when the copy of the counts
// did not arrive within the bounded wait.
// The scan is split in two so that the copy engines can issue their first
// row loads while the table is on its way: scan_tile_bases_begin (thread 0
// issues one bulk copy of the whole table, rounded up to 16 bytes: the
// table's region is padded to 256) and scan_tile_bases_end (every thread).
__shared__ __align__(8) uint64_t s_scan_bar;

__device__ __forceinline__ void scan_tile_bases_begin(const ScatterParams& p, int* s_base) {
    if (threadIdx.x == 0) {
        const uint32_t bar = smem_addr(&s_scan_bar);
        mbar_init(bar, 1u);
        mbar_fence_init();
        const uint32_t bytes = ((uint32_t)p.numTiles * (p.W + 1) * 4u + 15u) & ~15u;
        mbar_arrive_expect_tx(bar, bytes);
        bulk_load(smem_addr(s_base), p.tile_cnt, bytes, bar);
    }
}

__device__ int scan_tile_bases_end(const ScatterParams& p, int* s_base, int* rows) {
    __shared__ int s_tot[kMaxWorld + 1];
    const int C = p.W + 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const uint32_t bar = smem_addr(&s_scan_bar);
    __syncthreads();  // the barrier is initialised
    if (!__syncthreads_and(mbar_wait_bounded(bar, 0u))) {
        if (threadIdx.x == 0) atomicOr(p.err, EP_DEVERR_TIMEOUT);
        return -1;
    }
    for (int col = warp; col < C; col += nwarps) {
        int running = 0;
        for (int t0 = 0; t0 < p.numTiles; t0 += 32) {
            const int t = t0 + lane;
            const int v = t < p.numTiles ? s_base[t * C + col] : 0;
            int incl = v;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int m = __shfl_up_sync(kFull, incl, off);
                if (lane >= off) incl += m;
            }
            if (t < p.numTiles) s_base[t * C + col] = running + incl - v;
            running += __shfl_sync(kFull, incl, 31);
        }
        if (lane == 0) s_tot[col] = running;
    }
    __syncthreads();
    if (blockIdx.x == 0 && (int)threadIdx.x < p.W) {
        p.recv_count[threadIdx.x] = s_tot[threadIdx.x];  // stored, not accumulated
        if (s_tot[threadIdx.x] > p.maxRecv) atomicOr(p.err, EP_DEVERR_CAPACITY);
    }
    int r = 0;
    for (int pe = 0; pe < p.W; ++pe) r += s_tot[pe];
    *rows = r;
    return s_tot[p.W];
}

__device__ int scan_tile_bases(const ScatterParams& p, int* s_base, int* rows) {
    scan_tile_bases_begin(p, s_base);
    return scan_tile_bases_end(p, s_base, rows);
}

// =====================================================================
// Per-token bookkeeping of the scatter, done by one warp. The three global
// reads it needs (the routing row, the tile bases, the topk ids) do not depend
// on one another; TokenInputs holds them so that a warp can issue them for its
// next token before it works on the current one.
// =====================================================================
struct TokenInputs {
    int h;     // the feed's handle of the token, or -1 when nothing is loaded
    int g;     // token
    int2 rr;   // lane < W: (tile-local rank or -1, weight bits); OwnFeed: (slot, or -1 / -2, -)
    int base;  // lane < W: base of the token's tile at destination lane
    int e;     // lane < k: topk id
    float wt;  // lane < k: topk weight (list feed only)
};

// kSmemBase: the tile bases are in shared memory (s_base), else in global memory.
template <bool kSmemBase>
__device__ __forceinline__ TokenInputs load_token_inputs(const ScatterParams& p, int g, int lane,
                                                       const int* s_base) {
    TokenInputs in;
    in.h = g;
    in.g = g;
    in.wt = 0.0f;
    const int W = p.W;
    // routing data written by other blocks (or the previous kernel): read through L2
    in.rr = lane < W ? __ldcg(p.route + (size_t)g * W + lane) : make_int2(-1, 0);
    const size_t bi = (size_t)(g >> p.baseShift) * p.baseStride + lane;
    if (kSmemBase) in.base = lane < W ? s_base[bi] : 0;
    else in.base = lane < W ? __ldcg(p.tile_base + bi) : 0;
    in.e = lane < p.k ? p.idx[(size_t)g * p.k + lane] : -1;
    return in;
}

// Where the rows, meta records and scale rows of each destination start, for
// the kernels of one block: slot s of destination pe is at s_dst_x[pe] +
// s * rowBytes (and likewise for the records and scale rows), and slots at or
// above s_dst_cap[pe] are refused. On one GPU the destinations are regions of
// recv_x / recv_meta / recv_scales, pe * maxRecv rows apart. With ranks in
// separate processes each destination is another rank's receive buffer, where
// this rank's rows start after those of the ranks before it (the count table),
// so slots are counted from there.
__shared__ uint8_t* s_dst_x[kMaxWorld];
__shared__ int32_t* s_dst_meta[kMaxWorld];
__shared__ uint32_t* s_dst_scales[kMaxWorld];
__shared__ int s_dst_cap[kMaxWorld];
// Bounds-checking build: the end of each destination's receive rows, meta
// records and scale rows.
__shared__ const uint8_t* s_dst_x_end[kDebugBounds ? kMaxWorld : 1];
__shared__ const int32_t* s_dst_meta_end[kDebugBounds ? kMaxWorld : 1];
__shared__ const uint32_t* s_dst_scales_end[kDebugBounds ? kMaxWorld : 1];

// Bounds-checking build: false (and EP_DEVERR_BOUNDS) when [p, p + bytes)
// is not inside [lo, hi).
__device__ __forceinline__ bool in_bounds(const void* p, long long bytes, const void* lo, const void* hi, int32_t* err) {
    if (!kDebugBounds) return true;
    const char* a = static_cast<const char*>(p);
    if (a >= static_cast<const char*>(lo) && a + bytes <= static_cast<const char*>(hi)) return true;
    atomicOr(err, EP_DEVERR_BOUNDS);
    return false;
}

// Every thread of the block calls it (it ends with __syncthreads); with
// peers, after the count table is complete. Block 0 stores the rows this rank
// receives. Returns false when an earlier barrier of the call gave up: then
// nothing may be written to the other ranks.
__device__ __forceinline__ bool dest_setup(const ScatterParams& p) {
    const int pe = threadIdx.x;
    if (pe < p.W) {
        long long first;  // this source's first row in destination pe's buffers
        uint8_t* x;
        int32_t* meta;
        uint32_t* sc = nullptr;
        if (p.peers != nullptr) {
            int before = 0;
            for (int r = 0; r < p.rank; ++r) before += __ldcg(p.counts + r * p.W + pe);
            first = before;
            x = p.peers->recv_x[pe];
            meta = p.peers->recv_meta[pe];
        } else {
            first = (long long)pe * p.maxRecv;
            x = p.recv_x;
            meta = p.recv_meta;
            sc = p.recv_scales;
        }
        s_dst_x[pe] = x + first * p.rowBytes;
        s_dst_meta[pe] = meta + first * p.M;
        s_dst_scales[pe] = sc != nullptr ? sc + first * p.scaleWords : nullptr;
        s_dst_cap[pe] = p.peers != nullptr ? p.maxRecv - (int)first : p.maxRecv;
        if (kDebugBounds) {
            const long long end = (p.peers != nullptr ? 0 : (long long)pe * p.maxRecv) + p.boundsRows;
            s_dst_x_end[pe] = x + end * p.rowBytes;
            s_dst_meta_end[pe] = meta + end * p.M;
            s_dst_scales_end[pe] = sc != nullptr ? sc + end * p.scaleWords : nullptr;
        }
    }
    const bool go = __syncthreads_and(p.peers == nullptr || (__ldcg(p.err) & EP_DEVERR_TIMEOUT) == 0) != 0;
    if (go && p.peers != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
        int total = 0;
        for (int r = 0; r < p.W; ++r) total += __ldcg(p.counts + r * p.W + p.rank);
        *p.recv_total = total;
        if (total > p.maxRecv) atomicOr(p.err, EP_DEVERR_CAPACITY);
    }
    return go;
}

// The scale row of token g travels with it to every destination in `mask`
// (lane pe holds the slot at pe).
__device__ __forceinline__ void write_scales(const ScatterParams& p, int g, uint32_t mask, int my_slot, int lane) {
    const uint32_t* src = p.scales + (size_t)g * p.scaleWords;
    for (int w0 = 0; w0 < p.scaleWords; w0 += 32) {
        const int wi = w0 + lane;
        const uint32_t v = wi < p.scaleWords ? src[wi] : 0u;
        for (uint32_t m = mask; m; m &= m - 1) {
            const int pe = __ffs(m) - 1;
            const int slot = __shfl_sync(kFull, my_slot, pe);
            uint32_t* dst = s_dst_scales[pe] + (size_t)slot * p.scaleWords + wi;
            if (wi < p.scaleWords && in_bounds(dst, 4, s_dst_scales[pe], s_dst_scales_end[kDebugBounds ? pe : 0], p.err))
                *dst = v;
        }
    }
}

// Meta records and scale rows of token g at every destination in `mask`.
// Lane pe holds the token's slot at pe (my_slot) and its weight-sum bits
// (wb_lane); lane j < k holds topk id e of entry j.
__device__ __forceinline__ void write_records(const ScatterParams& p, int g, uint32_t mask, int my_slot,
                                              int wb_lane, int e, int lane) {
    const int r = p.peers != nullptr ? p.rank : g / p.T, t = g - (p.peers != nullptr ? 0 : r * p.T);
    const int pe_e = (e >= 0 && e < p.E) ? e / p.nEpr : -1;
    // field f of a record: 0 rank, 1 token, 2 weight bits, 3+j local id of entry j
    const int j0 = lane - 3, j1 = lane + 29;
    const int e0 = __shfl_sync(kFull, e, j0 & 31), q0 = __shfl_sync(kFull, pe_e, j0 & 31);
    const int e1 = __shfl_sync(kFull, e, j1 & 31), q1 = __shfl_sync(kFull, pe_e, j1 & 31);
    for (uint32_t m = mask; m; m &= m - 1) {
        const int pe = __ffs(m) - 1;
        const int slot = __shfl_sync(kFull, my_slot, pe);
        const int wb = __shfl_sync(kFull, wb_lane, pe);
        int32_t* rec = s_dst_meta[pe] + (size_t)slot * p.M;
        if (!in_bounds(rec, 4LL * p.M, s_dst_meta[pe], s_dst_meta_end[kDebugBounds ? pe : 0], p.err)) continue;
        int v0;
        if (lane == 0) v0 = r;
        else if (lane == 1) v0 = t;
        else if (lane == 2) v0 = wb;
        else v0 = (q0 == pe) ? e0 - pe * p.nEpr : -1;
        if (lane < p.M) rec[lane] = v0;
        if (lane + 32 < p.M) rec[lane + 32] = (q1 == pe) ? e1 - pe * p.nEpr : -1;
    }
    if (p.scaleWords > 0) write_scales(p, g, mask, my_slot, lane);
}

// Turn the tile-local ranks of the token into slots (lane pe holds the slot
// at pe), write them back into the routing table for combine, and write the
// token's meta record at every destination. Returns the destination mask.
__device__ __forceinline__ uint32_t token_slots_and_meta(const ScatterParams& p, const TokenInputs& in,
                                                         int lane, int& my_slot) {
    const int W = p.W, g = in.g;
    const int2 rr = in.rr;
    my_slot = -1;
    bool ok = false;
    if (rr.x >= 0) {
        my_slot = in.base + rr.x;
        ok = my_slot < s_dst_cap[lane];  // always, unless the counts were corrupted
        if (!ok) atomicOr(p.err, EP_DEVERR_CAPACITY);
        p.route[(size_t)g * W + lane].x = ok ? my_slot : -1;
    }
    const uint32_t mask = __ballot_sync(kFull, ok);
    write_records(p, g, mask, my_slot, rr.y, in.e, lane);
    return mask;
}

// =====================================================================
// scatter_rows (TMA): persistent copy engines, one per warp.
// Items are (present token, chunk) pairs of the tokens this engine's feed
// hands it; an S-stage ring keeps S - kPend loads ahead and lets kPend
// items' bulk stores drain while the next load starts.
// =====================================================================
template <int kPend>
__device__ __forceinline__ void bulk_wait_read_pend() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kPend) : "memory");
}

// Shared memory of the copy engines of one block, carved from the dynamic
// shared memory: [mbarriers: nwarps*S][ring: nwarps*S*2 int] pad 128 | stages.
struct EngineSmem {
    uint32_t stage0_addr;  // this warp's first stage
    uint32_t bar0;         // this warp's first mbarrier
    int* item_tok;         // [S] token of the item in each stage
    int* item_chunk;       // [S] row piece of the item in each stage
};

__device__ __forceinline__ EngineSmem engine_smem_init(uint8_t* smem, const ScatterParams& p, int warp,
                                                       int nwarps, int lane) {
    const int S = p.stages;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    int* ring = reinterpret_cast<int*>(smem + (size_t)nwarps * S * sizeof(uint64_t));
    const size_t head = ((size_t)nwarps * S * (sizeof(uint64_t) + 2 * sizeof(int)) + 127) & ~(size_t)127;
    EngineSmem es;
    es.stage0_addr = smem_addr(smem + head + (size_t)warp * S * p.chunkStride);
    es.bar0 = smem_addr(bars + warp * S);
    es.item_tok = ring + warp * S * 2;
    es.item_chunk = es.item_tok + S;
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(es.bar0 + 8u * s, 1u);
        mbar_fence_init();
    }
    __syncwarp();
    return es;
}

// Engines per block: at a high mean fan-out the copies are bandwidth-bound
// and one engine fewer per SM writes faster (B200: 472 vs 503 us at fan-out
// 5.3); at a low fan-out the per-token latency chain dominates and every
// engine helps (skewed routing, fan-out 2.9: 302 vs 335 us). The counts of
// this dispatch (recv_count, complete before the call) decide.
// rows: the call's rows at all destinations, or -1: read them from recv_count.
__device__ __forceinline__ int active_engines(const ScatterParams& p, int nwarps, int lane, int rows) {
    if (p.fanoutSwitch <= 0 || nwarps <= 2) return nwarps;
    if (rows < 0) {
        rows = lane < p.W ? __ldcg(p.recv_count + lane) : 0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) rows += __shfl_xor_sync(kFull, rows, off);
    }
    return (long long)rows * 100 > (long long)p.fanoutSwitch * p.G ? nwarps - 1 : nwarps;
}

// Token feeds of a copy engine. A feed hands out token handles (p.G: none
// left), maps a handle to the token's row, issues the global loads of a
// token's inputs (so that the engine can prefetch them one token ahead), and
// prepares a token: its slots, routing-table entries and meta records.

// Split dispatch feeds: route_count's tile-local ranks plus the tile's base
// give a token's slots. There is one feed per hand-out mode, each templated on
// where the tile bases live, so that the per-token path has no branch on
// either (the choice is made once per engine).

// Dense batches: tokens from the shared hand-out (static rounds, then a
// global counter). Two candidates are kept in flight ahead (the hand-out's
// answer and then the token's destination mask), so finding the next
// present token costs no latency on the copy path.
template <bool kSmemBase>
struct DynFeed {
    TokenSource src;
    int tA, tB, tC;  // candidates, in the order handed out (lane 0)
    uint32_t mA, mB;  // masks of A and B
    const int* s_base;

    __device__ __forceinline__ void init(const ScatterParams& p, const TokenSource& s0, int lane,
                                         const int* bases) {
        src = s0;
        s_base = bases;
        tA = tB = tC = p.G;
        mA = mB = 0u;
        if (lane == 0) {
            tA = source_next(src);
            tB = source_next(src);
            mA = tA < p.G ? __ldcg(p.tok_mask + tA) : 0u;
            tC = source_next(src);
            mB = tB < p.G ? __ldcg(p.tok_mask + tB) : 0u;
        }
    }
    // Next present token (warp-uniform), or p.G.
    __device__ __forceinline__ int next(const ScatterParams& p, int lane) {
        int found = p.G;
        if (lane == 0) {
            while (tA < p.G) {
                const int t = tA;
                const uint32_t m = mA;
                tA = tB;
                mA = mB;
                tB = tC;
                mB = tC < p.G ? __ldcg(p.tok_mask + tC) : 0u;
                tC = tC < p.G ? source_next(src) : p.G;
                if (m != 0u) {
                    found = t;
                    break;
                }
            }
        }
        return __shfl_sync(kFull, found, 0);
    }
    __device__ __forceinline__ int row(const ScatterParams&, int h) const { return h; }
    __device__ __forceinline__ TokenInputs load(const ScatterParams& p, int h, int lane) const {
        return load_token_inputs<kSmemBase>(p, h, lane, s_base);
    }
    __device__ __forceinline__ uint32_t prepare(const ScatterParams& p, const TokenInputs& in, int lane,
                                                int& my_slot) const {
        return token_slots_and_meta(p, in, lane, my_slot);
    }
};

// Sparse batches (fewer than 8 present tokens per worker): static hand-out
// only; the worker's rounds are scanned 32 at a time, lane l loading the
// mask of round i0 + l, and the next 32 masks are loaded while these are
// used.
template <bool kSmemBase>
struct StaticFeed {
    TokenSource src;
    int i0;
    uint32_t pm;     // present rounds of [i0, i0 + 32) not yet handed out
    uint32_t mnext;  // this lane's mask in the next 32 rounds
    const int* s_base;

    // Whether the token of round i is present, from its ids (an id in
    // [0, E)): the ids are an input of the call, so this needs nothing from
    // route_count and may run before the scatter waits for it.
    __device__ __forceinline__ uint32_t round_mask(const ScatterParams& p, int i) const {
        const long long t = src.w + (long long)i * src.nU;
        if (i >= src.R || t >= p.G) return 0u;
        const int32_t* ids = p.idx + (size_t)t * p.k;
        bool any = false;
        for (int j0 = 0; j0 < p.k; j0 += 8) {
            int e[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) e[j] = j0 + j < p.k ? ids[j0 + j] : -1;
#pragma unroll
            for (int j = 0; j < 8; ++j) any |= e[j] >= 0 && e[j] < p.E;
        }
        return any ? 1u : 0u;
    }
    __device__ __forceinline__ void init(const ScatterParams& p, const TokenSource& s0, int lane,
                                         const int* bases) {
        src = s0;
        s_base = bases;
        i0 = 0;
        const uint32_t m0 = round_mask(p, lane);
        mnext = round_mask(p, 32 + lane);
        pm = __ballot_sync(kFull, m0 != 0u);
    }
    __device__ __forceinline__ int next(const ScatterParams& p, int lane) {
        while (pm == 0u) {
            i0 += 32;
            if (i0 >= src.R) return p.G;
            pm = __ballot_sync(kFull, mnext != 0u);
            mnext = round_mask(p, i0 + 32 + lane);
        }
        const int l = __ffs(pm) - 1;
        pm &= pm - 1;
        return src.w + (i0 + l) * src.nU;
    }
    __device__ __forceinline__ int row(const ScatterParams&, int h) const { return h; }
    __device__ __forceinline__ TokenInputs load(const ScatterParams& p, int h, int lane) const {
        return load_token_inputs<kSmemBase>(p, h, lane, s_base);
    }
    __device__ __forceinline__ uint32_t prepare(const ScatterParams& p, const TokenInputs& in, int lane,
                                                int& my_slot) const {
        return token_slots_and_meta(p, in, lane, my_slot);
    }
};

// One copy engine (a warp): the present tokens its feed hands out are copied
// row piece by row piece through an S-stage shared-memory ring, S - kPend
// loads ahead, with kPend items' bulk stores left draining when a stage is
// refilled.
// `ready` runs once the engine has issued its first loads (its whole
// lookahead, or p.earlyIssue of them) and before any store; every thread of
// the block calls it, so it may hold a block-wide barrier. false: copy
// nothing, only drain the loads.
template <int kPend, class Feed, class Ready>
__device__ __forceinline__ void copy_engine(const ScatterParams& p, const EngineSmem& es, int lane, Feed& feed,
                                            Ready&& ready) {
    const int S = p.stages;  // > kPend (checked on the host)
    const uint32_t stage0_addr = es.stage0_addr, bar0 = es.bar0;
    int* item_tok = es.item_tok;
    int* item_chunk = es.item_chunk;

    int pg = feed.next(p, lane);  // producer token (handle)
    int pc = 0;                   // producer chunk
    int issued = 0, consumed = 0;
    bool ok = true;

    auto issue = [&]() {
        const int s = issued % S;
        if (lane == 0) {
            const long long off = (long long)pc * p.chunkBytes;
            const long long rem = p.rowBytes - off;
            const uint32_t bytes = (uint32_t)(rem < p.chunkBytes ? rem : p.chunkBytes);
            item_tok[s] = pg;
            item_chunk[s] = pc;
            const uint8_t* src = p.x + (size_t)feed.row(p, pg) * p.rowBytes + off;
            if (in_bounds(src, bytes, p.x, p.x + (size_t)p.G * p.rowBytes, p.err)) {
                mbar_arrive_expect_tx(bar0 + 8u * s, bytes);
                bulk_load(stage0_addr + (uint32_t)s * p.chunkStride, src, bytes, bar0 + 8u * s);
            } else {
                mbar_arrive(bar0 + 8u * s);  // the stage completes without data
            }
        }
        ++issued;
        if (++pc == p.numChunks) {
            pc = 0;
            pg = feed.next(p, lane);
        }
    };

    const int lookahead = S - kPend;
    // Loads issued before the ready hook: the whole lookahead, unless the
    // kernel caps them (earlyIssue > 0: at most that many; < 0: none).
    const int early = p.earlyIssue == 0 ? lookahead : min(lookahead, max(p.earlyIssue, 0));
    for (int i = 0; i < early && pg < p.G; ++i) issue();
    if (!ready()) {
        ok = false;
        pg = p.G;
    }
    while (ok && issued < lookahead && pg < p.G) issue();

    // Per-token state kept across the chunks of one token.
    TokenInputs pre;
    pre.h = -1;
    int cur_tok = -1;
    uint32_t cur_mask = 0;
    int my_slot = -1;  // lane pe: slot of the current token at pe

    while (ok && consumed < issued) {
        const int s = consumed % S;
        const uint32_t parity = (uint32_t)(consumed / S) & 1u;
        __syncwarp();
        const int h = item_tok[s];
        const int c = item_chunk[s];

        if (h != cur_tok) {
            cur_tok = h;
            const TokenInputs in = (pre.h == h) ? pre : feed.load(p, h, lane);
            // Prefetch the next token in the ring before working on this one.
            pre.h = -1;
            const int nxt = consumed + p.numChunks - c;
            if (nxt < issued) pre = feed.load(p, item_tok[nxt % S], lane);
            cur_mask = feed.prepare(p, in, lane, my_slot);
        }

        // Wait for the row piece, then send it to every destination.
        bool got = true;
        if (lane == 0) got = mbar_wait_bounded(bar0 + 8u * s, parity);
        got = __shfl_sync(kFull, got, 0) != 0;
        if (!got) {
            ok = false;
            break;
        }
        const long long off = (long long)c * p.chunkBytes;
        const long long rem = p.rowBytes - off;
        const uint32_t bytes = (uint32_t)(rem < p.chunkBytes ? rem : p.chunkBytes);
        for (uint32_t m = cur_mask; m; m &= m - 1) {
            const int pe = __ffs(m) - 1;
            const int slot = __shfl_sync(kFull, my_slot, pe);
            uint8_t* dst = s_dst_x[pe] + (size_t)slot * p.rowBytes + off;
            if (lane == 0 && in_bounds(dst, bytes, s_dst_x[pe], s_dst_x_end[kDebugBounds ? pe : 0], p.err))
                bulk_store(dst, stage0_addr + (uint32_t)s * p.chunkStride, bytes);
        }
        if (lane == 0) bulk_commit();
        ++consumed;

        // Refill the stage whose stores (kPend items back) have been read out.
        if (pg < p.G) {
            if (lane == 0) bulk_wait_read_pend<kPend>();
            __syncwarp();
            issue();
        }
    }

    if (!ok) {
        // Give up: record it, then drain what this engine still has in flight.
        if (lane == 0) {
            atomicOr(p.err, EP_DEVERR_TIMEOUT);
            for (int i = consumed; i < issued; ++i)
                mbar_wait_bounded(bar0 + 8u * (i % S), (uint32_t)(i / S) & 1u);
        }
    }
    if (lane == 0) bulk_wait_all();
    // Another rank reads these rows after a barrier: make this engine's bulk
    // stores visible beyond this GPU first.
    if (p.peers != nullptr && lane == 0) {
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence_system();
    }
    __syncwarp();
}

// One split-dispatch copy engine, with the feed of the call's hand-out mode.
template <int kPend, bool kSmemBase>
__device__ __forceinline__ void run_split_engine(const ScatterParams& p, const EngineSmem& es, int lane,
                                                 const TokenSource& src, const int* s_base) {
    if (src.dyn) {
        DynFeed<kSmemBase> feed;
        feed.init(p, src, lane, s_base);
        copy_engine<kPend>(p, es, lane, feed, [] { return true; });
    } else {
        StaticFeed<kSmemBase> feed;
        feed.init(p, src, lane, s_base);
        copy_engine<kPend>(p, es, lane, feed, [] { return true; });
    }
}

// Split-dispatch copy engines: the engines of this block that the fan-out
// leaves active take tokens from the shared hand-out. P: present tokens of
// the call; rows: its rows at all destinations (-1: read recv_count);
// s_base: tile bases in shared memory, or nullptr.
template <int kPend>
__device__ __forceinline__ void global_copy_engines(const ScatterParams& p, const EngineSmem& es, int lane,
                                                    int warp, int nwarps, int P, int rows, const int* s_base) {
    const int engines = active_engines(p, nwarps, lane, rows);
    if (warp >= engines) return;  // this engine's stages stay unused
    const TokenSource src = make_source(warp * gridDim.x + blockIdx.x, gridDim.x * engines, p.G, p.work, P);
    if (s_base != nullptr) run_split_engine<kPend, true>(p, es, lane, src, s_base);
    else run_split_engine<kPend, false>(p, es, lane, src, nullptr);
}

// Shared memory: the copy engines' barriers, rings and stages at
// engineOffset, and the tile bases (when the scatter scans them) at
// baseOffset. kDense: the instance for large batches, whose copy engines only
// take the shared hand-out with tile bases from global memory (one code path,
// as compact as the loop allows); the other instance also has the sparse
// hand-out and the shared-memory tile bases.
template <int kPend, bool kDense>
__global__ void __launch_bounds__(kMaxScatterWarps * 32) ep_scatter_rows_kernel(ScatterParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    if (kDense) {
        const EngineSmem es = engine_smem_init(smem, p, warp, nwarps, lane);
        pdl_wait();     // routing written by route_count is visible from here on
        if (!dest_setup(p)) return;
        const int engines = active_engines(p, nwarps, lane, -1);
        if (warp >= engines) return;  // this engine's stages stay unused
        DynFeed<false> feed;
        feed.init(p, make_source(warp * gridDim.x + blockIdx.x, gridDim.x * engines, p.G, p.work, p.G), lane,
                  nullptr);
        copy_engine<kPend>(p, es, lane, feed, [] { return true; });
        return;
    }
    int* s_base = p.baseSmemBytes > 0 ? reinterpret_cast<int*>(smem + p.baseOffset) : nullptr;
    const EngineSmem es = engine_smem_init(smem + p.engineOffset, p, warp, nwarps, lane);
    const int nAll = gridDim.x * nwarps;
    if (s_base != nullptr && p.G < 8 * nAll) {
        // Fewer than 8 tokens per engine: the hand-out is static whatever the
        // counts say, so every engine starts at once (all of them: the
        // fan-out switch would need the counts). It finds its tokens from
        // their ids and issues their first row loads before waiting for
        // route_count: x and the ids come from work that finished before
        // route_count could start, and this kernel only launches once
        // route_count has passed its own wait. The wait, the copy of the
        // tile counts and their scan complete before the first store.
        StaticFeed<true> feed;
        feed.init(p, make_source(warp * gridDim.x + blockIdx.x, nAll, p.G, p.work, 0), lane, s_base);
        int rows;
        copy_engine<kPend>(p, es, lane, feed, [&] {
            pdl_wait();  // routing written by route_count is visible from here on
            if (!dest_setup(p)) return false;
            scan_tile_bases_begin(p, s_base);
            return scan_tile_bases_end(p, s_base, &rows) >= 0;
        });
        return;
    }
    pdl_wait();     // routing written by route_count is visible from here on
    if (!dest_setup(p)) return;
    int P, rows = -1;
    if (s_base != nullptr) {
        P = scan_tile_bases(p, s_base, &rows);
        if (P < 0) return;  // the counts did not arrive: nothing is copied
    } else {
        P = p.ptotal != nullptr ? __ldcg(p.ptotal) : p.G;
    }
    global_copy_engines<kPend>(p, es, lane, warp, nwarps, P, rows, s_base);
}

__device__ __forceinline__ int dest_pe(int e, int nEpr, int shift) { return shift >= 0 ? e >> shift : e / nEpr; }

// =====================================================================
// dispatch_fused: the whole dispatch of a small batch in one launch. Block b
// owns the tokens [lo, hi) of an even, contiguous split of the batch (every
// block owns at least one), routes them and copies them itself:
//   1. the chunks of 32 tokens holding own tokens: destination masks (shared
//      memory) and, per chunk and destination, the own tokens that go there;
//      the own tokens' ids and weights (shared memory); the present own
//      tokens form a list;
//   2. the block publishes its totals per destination in words tagged with
//      the call's epoch (decoupled look-back, as in single-pass prefix
//      scans); each copy-engine warp issues the row load of its first present
//      own token;
//   3. every thread adds up a share of the earlier blocks' words, each loaded
//      once its tag shows this call (a bounded wait: blocks publish before
//      they wait and wait only on lower-numbered ones, so the waits end), into
//      the block's base at each destination; slots of the own tokens (base +
//      rank among the own tokens going there; -1: not sent there, -2: beyond
//      maxRecv); routing rows of the absent own tokens; the last block stores
//      recv_count;
//   4. the engines copy the present own tokens, handed out through a
//      shared-memory counter: per token its routing row and meta records (and
//      scale rows), then the row's bulk stores.
// A block's word q holds its totals at destinations 6q .. 6q+5 (8 bits each:
// a block owns at most kFusedMaxOwn < 256 tokens) under a 16-bit tag, so that
// one 64-bit load brings a count and the proof that it is this call's. The
// epoch advances once every block has read it (the last block to get past
// its look-back), so replays of a captured graph stay in step.
// Shared memory: the routing area (FusedLayout) at 0, the copy engines'
// barriers and stages at engineOffset.
// =====================================================================
constexpr int kFusedPerWord = 6;

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Destination mask of token g from its ids (ids outside [0, E) are masked;
// `bad` reports ids >= E); its k ids and weights (0 without weights) are also
// kept in sid / sw for the copy engines. All loads are issued before any is
// used.
template <int kK>
__device__ __forceinline__ uint32_t token_dest_mask(const ScatterParams& p, int g, bool& bad, int* sid, float* sw) {
    const int32_t* ids = p.idx + (size_t)g * p.k;
    const float* wts = p.w != nullptr ? p.w + (size_t)g * p.k : nullptr;
    int e[kK];
    float w[kK];
#pragma unroll
    for (int j = 0; j < kK; ++j) {
        e[j] = j < p.k ? ids[j] : -1;
        w[j] = (j < p.k && wts != nullptr) ? wts[j] : 0.0f;
    }
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < kK; ++j) {
        if (j < p.k) {
            sid[j] = e[j];
            sw[j] = w[j];
        }
        if (e[j] >= p.E) bad = true;
        if (e[j] >= 0 && e[j] < p.E) m |= 1u << dest_pe(e[j], p.nEpr, p.nEprShift);
    }
    return m;
}

// The own tokens' feed: list entry i (a present own token) is handle i.
struct OwnFeed {
    const int* list;  // present own tokens, ascending
    int* ctr;         // next entry to hand out (shared memory)
    const int* slot;  // [own][W]: slot of own token g - lo at each destination
    const int* ids;   // [own][k]: its topk ids, and weights
    const float* wts;
    int n, lo;

    __device__ __forceinline__ int next(const ScatterParams& p, int lane) {
        int i = 0;
        if (lane == 0) i = atomicAdd(ctr, 1);
        i = __shfl_sync(kFull, i, 0);
        return i < n ? i : p.G;
    }
    __device__ __forceinline__ int row(const ScatterParams&, int h) const { return list[h]; }
    __device__ __forceinline__ TokenInputs load(const ScatterParams& p, int h, int lane) const {
        TokenInputs in;
        in.h = h;
        in.g = list[h];
        in.rr = make_int2(lane < p.W ? slot[(in.g - lo) * p.W + lane] : -1, 0);
        in.base = 0;
        in.e = lane < p.k ? ids[(in.g - lo) * p.k + lane] : -1;
        in.wt = lane < p.k ? wts[(in.g - lo) * p.k + lane] : 0.0f;
        return in;
    }
    // Lane pe: the token's weight sum at pe (float32, topk order), its routing
    // row and, for every destination it reaches, its meta record.
    __device__ __forceinline__ uint32_t prepare(const ScatterParams& p, const TokenInputs& in, int lane,
                                                int& my_slot) const {
        const int pe_e = (in.e >= 0 && in.e < p.E) ? dest_pe(in.e, p.nEpr, p.nEprShift) : -1;
        float ws = 0.0f;
        for (int j = 0; j < p.k; ++j) {
            const int q = __shfl_sync(kFull, pe_e, j);
            const float wj = __shfl_sync(kFull, in.wt, j);
            if (q == lane) ws = ws + wj;
        }
        const int s = in.rr.x;
        my_slot = s >= 0 ? s : -1;
        const int wb = s != -1 ? __float_as_int(p.useWeights ? ws : 1.0f) : 0;
        if (lane < p.W) p.route[(size_t)in.g * p.W + lane] = make_int2(my_slot, wb);
        const uint32_t mask = __ballot_sync(kFull, my_slot >= 0);
        write_records(p, in.g, mask, my_slot, wb, in.e, lane);
        return mask;
    }
};

template <int kW, int kK>
__global__ void __launch_bounds__(kFusedWarps * 32, 1) ep_dispatch_fused_kernel(ScatterParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_base[kW];
    __shared__ unsigned s_tag;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int G = p.G, W = p.W, b = blockIdx.x;
    const int lo = (int)((long long)b * G / gridDim.x);
    const int hi = (int)((long long)(b + 1) * G / gridDim.x);  // > lo: the grid has at most G blocks
    const FusedLayout L = fused_layout(p.fusedOwn, W, nwarps, p.k);
    uint32_t* cmask = reinterpret_cast<uint32_t*>(smem + L.cmask);
    int* ccnt = reinterpret_cast<int*>(smem + L.ccnt);
    int* slot = reinterpret_cast<int*>(smem + L.slot);
    int* list = reinterpret_cast<int*>(smem + L.list);
    int* ctr = reinterpret_cast<int*>(smem + L.ctr);
    int* sids = reinterpret_cast<int*>(smem + L.ids);
    float* swts = reinterpret_cast<float*>(smem + L.wts);
    const int c_lo = lo >> 5, nch = ((hi + 31) >> 5) - c_lo;
    const int nw = (W + kFusedPerWord - 1) / kFusedPerWord;  // words per block

    pdl_wait();  // the ids, x and the previous call's words are visible from here on
    if (tid == 0) s_tag = ((__ldcg(p.fused_epoch) << 1) | 1u) & 0xffffu;
    if (tid < kW) s_base[tid] = 0;

    // 1. Masks of the own chunks' tokens; own tokens per chunk and destination.
    for (int i = warp; i < nch; i += nwarps) {
        const int g = (c_lo + i) * 32 + lane;
        const bool own = g >= lo && g < hi;
        bool bad = false;
        const uint32_t m = own ? token_dest_mask<kK>(p, g, bad, sids + (g - lo) * p.k, swts + (g - lo) * p.k) : 0u;
        if (bad) atomicOr(p.err, EP_DEVERR_EXPERT_RANGE);
        cmask[i * 32 + lane] = m;
#pragma unroll
        for (int pe = 0; pe < kW; ++pe) {
            if (pe < W) {
                const uint32_t bb = __ballot_sync(kFull, (m >> pe) & 1u);
                if (lane == pe) ccnt[i * W + pe] = __popc(bb);
            }
        }
    }
    dest_setup(p);  // ends with a block barrier (one GPU: always goes ahead)

    // 2. Publish this block's totals; list the present own tokens.
    if (warp == 0) {
        int tot = 0;
        if (lane < W)
            for (int i = 0; i < nch; ++i) tot += ccnt[i * W + lane];
        const unsigned tag = s_tag;
        for (int q = 0; q < nw; ++q) {
            unsigned long long v = tag;
#pragma unroll
            for (int u = 0; u < kFusedPerWord; ++u) {
                const int c = __shfl_sync(kFull, tot, (q * kFusedPerWord + u) & 31);
                if (q * kFusedPerWord + u < W) v |= (unsigned long long)c << (16 + 8 * u);
            }
            if (lane == 0) st_relaxed_u64(p.fused_agg + (size_t)b * nw + q, v);
        }
        if (hi == G && lane < W) ctr[2 + lane] = tot;  // the last block's own totals, for recv_count
        const int own = hi - lo, off = lo - c_lo * 32;
        int n = 0;
        for (int j0 = 0; j0 < own; j0 += 32) {
            const int j = j0 + lane;
            const bool present = j < own && cmask[off + j] != 0u;
            const uint32_t bb = __ballot_sync(kFull, present);
            if (present) list[n + __popc(bb & lanemask_lt())] = lo + j;
            n += __popc(bb);
        }
        if (lane == 0) {
            ctr[0] = n;
            ctr[1] = 0;
        }
    }
    __syncthreads();

    // 3; every thread of the block runs this once (the engines after issuing
    // their first row loads).
    auto route_rest = [&]() -> bool {
        const unsigned want = (s_tag + (p.barrierSlack << 1)) & 0xffffu;
        const int words = b * nw;
        int ok = 1;
        for (int i0 = 0; i0 < words; i0 += 4 * (int)blockDim.x) {
            unsigned long long v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * blockDim.x + tid;
                v[u] = i < words ? ld_relaxed_u64(p.fused_agg + i) : 0ull;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * blockDim.x + tid;
                if (i >= words) continue;
                if ((unsigned)(v[u] & 0xffffu) != want) {  // not yet published: wait, bounded
                    const long long t0 = clock64();
                    do {
                        if (clock64() - t0 > kWaitCycles) {
                            ok = 0;
                            break;
                        }
                        __nanosleep(32);
                        v[u] = ld_relaxed_u64(p.fused_agg + i);
                    } while ((unsigned)(v[u] & 0xffffu) != want);
                    if (!ok) break;
                }
                const int q = i % nw;
#pragma unroll
                for (int c = 0; c < kFusedPerWord; ++c) {
                    const int pe = q * kFusedPerWord + c;
                    const int n = (int)((v[u] >> (16 + 8 * c)) & 0xffu);
                    if (pe < W && n != 0) atomicAdd(&s_base[pe], n);
                }
            }
            if (!ok) break;
        }
        if (tid == 0 && atomicAdd(p.fused_done, 1u) == gridDim.x - 1) {
            *p.fused_done = 0u;  // every block has read the epoch: the next call's
            atomicAdd(p.fused_epoch, 1u);
        }
        if (!__syncthreads_and(ok)) {
            if (tid == 0) atomicOr(p.err, EP_DEVERR_TIMEOUT);
            return false;  // the bases are unknown: nothing is copied
        }
        if (warp == 0 && lane < W) {
            int run = s_base[lane];
            if (hi == G) {
                const int total = run + ctr[2 + lane];
                p.recv_count[lane] = total;  // stored, not accumulated
                if (total > p.maxRecv) atomicOr(p.err, EP_DEVERR_CAPACITY);
            }
            for (int i = 0; i < nch; ++i) {
                const int c = ccnt[i * W + lane];
                ccnt[i * W + lane] = run;
                run += c;
            }
        }
        __syncthreads();
        const uint32_t lt = lanemask_lt();
        for (int i = warp; i < nch; i += nwarps) {
            const int g = (c_lo + i) * 32 + lane;
            const uint32_t m = cmask[i * 32 + lane];  // 0 for tokens that are not own
            const bool own = g >= lo && g < hi;
#pragma unroll
            for (int pe = 0; pe < kW; ++pe) {
                if (pe < W) {
                    const bool hit = (m >> pe) & 1u;
                    const uint32_t bb = __ballot_sync(kFull, hit);
                    if (own) {
                        int sl = -1;
                        if (hit) {
                            sl = ccnt[i * W + pe] + __popc(bb & lt);
                            if (sl >= p.maxRecv) {  // only when maxRecv is exceeded
                                atomicOr(p.err, EP_DEVERR_CAPACITY);
                                sl = -2;
                            }
                        }
                        slot[(g - lo) * W + pe] = sl;
                        if (m == 0u) p.route[(size_t)g * W + pe] = make_int2(-1, 0);  // absent: no engine sees it
                    }
                }
            }
        }
        __syncthreads();
        return true;
    };

    // 4. The copies: each engine issues its first row load (p.earlyIssue) before
    // it joins the look-back, the rest once the slots are known.
    if (warp < p.fusedEngines) {
        const EngineSmem es = engine_smem_init(smem + p.engineOffset, p, warp, p.fusedEngines, lane);
        OwnFeed feed;
        feed.list = list;
        feed.ctr = ctr + 1;
        feed.slot = slot;
        feed.ids = sids;
        feed.wts = swts;
        feed.n = ctr[0];
        feed.lo = lo;
        copy_engine<1>(p, es, lane, feed, route_rest);
    } else {
        route_rest();
    }
}

// =====================================================================
// combine: one warp per token, 16-byte columns, fma fold in destPe order.
// =====================================================================

__device__ __forceinline__ void fma_bf16x8(float* acc, float w, const uint4& v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __uint_as_float(u[i] << 16);
        const float hi = __uint_as_float(u[i] & 0xffff0000u);
        acc[2 * i] = __fmaf_rn(w, lo, acc[2 * i]);
        acc[2 * i + 1] = __fmaf_rn(w, hi, acc[2 * i + 1]);
    }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float* acc) {
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __float22bfloat162_rn(make_float2(acc[2 * i], acc[2 * i + 1]));
        u[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint4(u[0], u[1], u[2], u[3]);
}

// Element types of the combine leg: bf16 in and out (float32 fold, RNE at the
// end), or float32 in and out (float32 fold, no final rounding).
struct CombineBf16 {
    static constexpr int kPer = 8;  // elements per 16-byte vector
    static __device__ __forceinline__ void fma(float* acc, float w, const uint4& v) { fma_bf16x8(acc, w, v); }
    static __device__ __forceinline__ uint4 pack(const float* acc) { return pack_bf16x8(acc); }
};

struct CombineF32 {
    static constexpr int kPer = 4;
    static __device__ __forceinline__ void fma(float* acc, float w, const uint4& v) {
        acc[0] = __fmaf_rn(w, __uint_as_float(v.x), acc[0]);
        acc[1] = __fmaf_rn(w, __uint_as_float(v.y), acc[1]);
        acc[2] = __fmaf_rn(w, __uint_as_float(v.z), acc[2]);
        acc[3] = __fmaf_rn(w, __uint_as_float(v.w), acc[3]);
    }
    static __device__ __forceinline__ uint4 pack(const float* acc) {
        return make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                          __float_as_uint(acc[3]));
    }
};

// One token's output row: for each group of kU 16-byte columns per lane, the
// loads of up to kB destination rows are issued together, then folded in
// destination order (so the result does not depend on kU, kB or kWide).
// kWide: a lane's columns come in adjacent pairs, each pair one 32-byte load
// (rows 32-byte aligned, V even: checked on the host).
template <class Elem, int kU, int kB, bool kWide>
__device__ __forceinline__ void combine_columns(const uint8_t* const* rows, const float* wts, int n, uint4* orow,
                                                int V, int lane) {
    constexpr int kP = kWide ? 2 : 1;  // 16-byte columns per load
    constexpr int kL = kU / kP;        // loads per lane and row in a pass
    static_assert(kU % kP == 0, "kU must be a multiple of the load width");
    const int VL = V / kP;             // loads across a row
    for (int v0 = lane; v0 < VL; v0 += 32 * kL) {
        float acc[kL][kP][Elem::kPer];
#pragma unroll
        for (int u = 0; u < kL; ++u)
#pragma unroll
            for (int h = 0; h < kP; ++h)
#pragma unroll
                for (int i = 0; i < Elem::kPer; ++i) acc[u][h][i] = 0.0f;
        for (int b = 0; b < n; b += kB) {
            uint4 val[kL][kB][kP];
#pragma unroll
            for (int i = 0; i < kB; ++i) {
                if (b + i < n) {
                    const uint8_t* row = rows[b + i];
#pragma unroll
                    for (int u = 0; u < kL; ++u) {
                        const int v = v0 + 32 * u;
                        if (v < VL) {
                            if constexpr (kWide) ld_stream_v8(row + (size_t)v * 32, val[u][i][0], val[u][i][kP - 1]);
                            else val[u][i][0] = ld_stream_v4(row + (size_t)v * 16);
                        }
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < kB; ++i) {
                if (b + i < n) {
                    const float w = wts[b + i];
#pragma unroll
                    for (int u = 0; u < kL; ++u)
                        if (v0 + 32 * u < VL)
#pragma unroll
                            for (int h = 0; h < kP; ++h) Elem::fma(acc[u][h], w, val[u][i][h]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kL; ++u) {
            const int v = v0 + 32 * u;
            if (v < VL)
#pragma unroll
                for (int h = 0; h < kP; ++h) orow[v * kP + h] = Elem::pack(acc[u][h]);
        }
    }
}

// kCols x kRows loads in flight per lane and pass; kMinBlocks blocks of 256
// threads per SM bound the registers (65536 / (256 * kMinBlocks)).
template <class Elem, int kCols, int kRows, int kMinBlocks, bool kWide>
__global__ void __launch_bounds__(kMaxCombineWarps * 32, kMinBlocks) ep_combine_kernel(CombineParams p) {
    __shared__ const uint8_t* s_row[kMaxCombineWarps][kMaxWorld];
    __shared__ float s_w[kMaxCombineWarps][kMaxWorld];
    pdl_wait();  // y and the routing of the dispatch are visible from here on
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int V = (int)(p.rowBytes / 16);
    const int W = p.W;

    // Lane pe: where destination pe's rows start in y. One GPU: region pe of
    // [W][maxRecv]. Ranks in processes: y is this rank's landing rows, in
    // destination order (this rank's count row gives each destination's rows).
    const uint8_t* ybase;
    if (p.counts != nullptr) {
        if ((__ldcg(p.err) & EP_DEVERR_TIMEOUT) != 0) return;  // a barrier of this call gave up
        const int c = lane < W ? __ldcg(p.counts + p.rank * W + lane) : 0;
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int m = __shfl_up_sync(kFull, incl, off);
            if (lane >= off) incl += m;
        }
        ybase = p.y + (size_t)(incl - c) * p.rowBytes;
    } else {
        ybase = p.y + (size_t)lane * p.maxRecv * p.rowBytes;
    }

    // Tokens come from the shared hand-out (a token's cost grows with its
    // number of destinations, so a purely static split would leave a tail);
    // the next token and its routing row are fetched one token ahead.
    TokenSource src = make_source(warp * gridDim.x + blockIdx.x, gridDim.x * (blockDim.x >> 5),
                                  p.G, p.work, p.G, 4);
    int next = 0;
    if (lane == 0) next = source_next(src);
    int g = __shfl_sync(kFull, next, 0);
    int2 rr_next = (g < p.G && lane < W) ? p.route[(size_t)g * W + lane] : make_int2(-1, 0);
    while (g < p.G) {
        const int2 rr = rr_next;
        if (lane == 0) next = source_next(src);
        const int g_next = __shfl_sync(kFull, next, 0);
        rr_next = (g_next < p.G && lane < W) ? p.route[(size_t)g_next * W + lane] : make_int2(-1, 0);

        const uint32_t mask = __ballot_sync(kFull, rr.x >= 0);
        uint4* orow = reinterpret_cast<uint4*>(p.out + (size_t)g * p.rowBytes);
        if (mask == 0u) {
            for (int v = lane; v < V; v += 32) orow[v] = make_uint4(0, 0, 0, 0);
            g = g_next;
            continue;
        }
        // Present destinations in ascending order: rank of this lane's bit.
        const int n = __popc(mask);
        if (rr.x >= 0) {
            const int pos = __popc(mask & lanemask_lt());
            const uint8_t* row = ybase + (size_t)rr.x * p.rowBytes;
            if (!in_bounds(row, p.rowBytes, p.y, p.y + p.yBytes, p.err)) row = p.y;  // skipped: reads y's first row
            s_row[warp][pos] = row;
            s_w[warp][pos] = __int_as_float(rr.y);
        }
        __syncwarp();

        combine_columns<Elem, kCols, kRows, kWide>(s_row[warp], s_w[warp], n, orow, V, lane);
        __syncwarp();
        g = g_next;
    }

    // The last block to finish resets the counter for the next combine (only
    // needed when the hand-out used it: the same for every block of a launch).
    if (!src.dyn) return;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(p.done, 1u) == gridDim.x - 1) {
            *p.work = 0;
            *p.done = 0u;
            __threadfence();
        }
    }
}

// =====================================================================
// Ranks in separate processes (one GPU each). Every rank maps every rank's
// shared buffers (receive rows, meta records, landing rows, count table,
// barrier flags); the PeerTable holds the addresses in this process.
// =====================================================================
__device__ __forceinline__ void st_release_sys_u32(unsigned* p, unsigned v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_sys_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// The barrier of the ranks, one warp. Each rank counts its barriers (the
// epoch lives on the device, so the replays of a captured graph stay in
// step, as the design page's cross-device barrier does); a rank arrives by
// storing its epoch in slot `rank` of every rank's flags, after a system-scope
// fence so that all it wrote before is visible to them, and then waits until
// every slot of its own flags has reached the epoch. The wait gives up after
// kWaitCycles and reports EP_DEVERR_TIMEOUT; the epochs of the ranks are then
// out of step and the communicator must be rebuilt.
__device__ __forceinline__ bool comm_barrier(const SyncParams& p, int lane) {
    unsigned e = 0;
    if (lane == 0) e = *p.epoch + 1u;
    e = __shfl_sync(kFull, e, 0);
    __threadfence_system();
    __syncwarp();
    if (lane < p.W) st_release_sys_u32(p.peers->flags[lane] + p.rank, e);
    bool ok = true;
    if (lane < p.W) {
        const unsigned* f = p.peers->flags[p.rank] + lane;
        const unsigned want = e + p.slack;
        if ((int)(ld_acquire_sys_u32(f) - want) < 0) {
            const long long t0 = clock64();
            while ((int)(ld_acquire_sys_u32(f) - want) < 0) {
                if (clock64() - t0 > kWaitCycles) {
                    ok = false;
                    break;
                }
                __nanosleep(64);
            }
        }
    }
    ok = __all_sync(kFull, ok);
    if (lane == 0) {
        *p.epoch = e;
        if (!ok) atomicOr(p.err, EP_DEVERR_TIMEOUT);
    }
    __threadfence_system();
    return ok;
}

// W ranks emulated by the W blocks of one cooperative launch (so that all of
// them run at once): rank r writes its word of round i, passes the barrier,
// then reads every rank's word of round i, which the barrier must have made
// visible. Rank `absent` stops arriving from round absentFrom on; the others
// must then give up (bounded wait) with EP_DEVERR_TIMEOUT.
__global__ void __launch_bounds__(32) ep_comm_barrier_test_kernel(BarrierTestParams p) {
    const int r = blockIdx.x, lane = threadIdx.x;
    SyncParams sp{};
    sp.peers = p.peers;
    sp.epoch = p.epochs + r;
    sp.err = p.errs + r;
    sp.rank = r;
    sp.W = p.W;
    int done = 0, bad = 0;
    for (int i = 0; i < p.rounds; ++i) {
        if (r == p.absent && i >= p.absentFrom) break;
        if (lane == 0) *reinterpret_cast<volatile int32_t*>(p.data + (size_t)r * p.rounds + i) = i + 1;
        if (!comm_barrier(sp, lane)) break;
        ++done;
        if (lane < p.W && *reinterpret_cast<volatile int32_t*>(p.data + (size_t)lane * p.rounds + i) != i + 1)
            ++bad;
    }
    for (int off = 16; off > 0; off >>= 1) bad += __shfl_xor_sync(kFull, bad, off);
    if (lane == 0) {
        p.rounds_done[r] = done;
        p.violations[r] = bad;
    }
}

__global__ void __launch_bounds__(32) ep_comm_sync_kernel(SyncParams p) {
    pdl_wait();  // the count row and the rows of the previous kernel are complete
    const int lane = threadIdx.x;
    if ((__ldcg(p.err) & EP_DEVERR_TIMEOUT) != 0) return;  // an earlier barrier gave up
    if (p.exchange && lane < p.W) {
        int32_t* dst = p.peers->counts[lane] + p.rank * p.W;
        for (int pe = 0; pe < p.W; ++pe) dst[pe] = __ldcg(p.myCount + pe);
    }
    if (p.barrier) comm_barrier(p, lane);
}

// The push: receive slot s of this rank holds a row of source r (slots are
// in source order, r's rows from before(r) on); its expert output goes to
// landing row land(r) + s - before(r) of rank r, where land(r) counts the
// rows r sent to the ranks before this one, so that r's landing rows are in
// destination order. One warp per row, 8 16-byte loads in flight per lane.
__global__ void __launch_bounds__(256) ep_comm_push_kernel(PushParams p) {
    __shared__ int s_before[kMaxWorld + 1];
    __shared__ int s_land[kMaxWorld];
    __shared__ uint8_t* s_dst[kMaxWorld];
    pdl_wait();  // the expert outputs and the count table are complete
    if ((__ldcg(p.err) & EP_DEVERR_TIMEOUT) != 0) return;  // a barrier gave up: touch no other rank
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    if (warp == 0) {
        const int c = lane < p.W ? __ldcg(p.counts + lane * p.W + p.rank) : 0;
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int m = __shfl_up_sync(kFull, incl, off);
            if (lane >= off) incl += m;
        }
        if (lane < p.W) {
            s_before[lane] = incl - c;
            int land = 0;
            for (int pe = 0; pe < p.rank; ++pe) land += __ldcg(p.counts + lane * p.W + pe);
            s_land[lane] = land;
            s_dst[lane] = p.peers->landing[lane];
        }
        if (lane == 31) s_before[p.W] = incl;
    }
    __syncthreads();
    const int total = s_before[p.W];
    if (total > p.maxRecv) {  // only when the counts were corrupted
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(p.err, EP_DEVERR_CAPACITY);
        return;
    }
    const int V = (int)(p.rowBytes / 16);
    for (int s = blockIdx.x * nwarps + warp; s < total; s += gridDim.x * nwarps) {
        int r = 0;
        while (r + 1 < p.W && s >= s_before[r + 1]) ++r;
        const long long li = (long long)s_land[r] + (s - s_before[r]);
        if (li >= p.maxLanding) {  // only when the counts were corrupted
            if (lane == 0) atomicOr(p.err, EP_DEVERR_CAPACITY);
            continue;
        }
        const uint8_t* src = p.y + (size_t)s * p.rowBytes;
        uint8_t* dst = s_dst[r] + (size_t)li * p.rowBytes;
        for (int v0 = lane; v0 < V; v0 += 32 * 8) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (v0 + 32 * u < V) v[u] = ld_stream_v4(src + (size_t)(v0 + 32 * u) * 16);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (v0 + 32 * u < V) *reinterpret_cast<uint4*>(dst + (size_t)(v0 + 32 * u) * 16) = v[u];
        }
    }
    __threadfence_system();  // the rows are read by rank r after the next barrier
}

}  // namespace

// ------------------------------------------------------------- launchers
namespace {
// Launch with programmatic stream serialisation (see pdl_wait / pdl_trigger).
template <typename P>
cudaError_t launch_pdl(void (*kernel)(P), int grid, int block, size_t smem, cudaStream_t s, const P& p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}
}  // namespace

// Instances by bounds on W and k (8, 16 or 32 each).
namespace {
template <bool kDense>
cudaError_t launch_route_count_as(const RouteParams& p, cudaStream_t s) {
    auto go = [&](auto kernel) { return launch_pdl(kernel, p.numTiles, kCountTile, 0, s, p); };
    if (p.W <= 8)
        return p.k <= 8    ? go(ep_route_count_kernel<8, 8, kDense>)
               : p.k <= 16 ? go(ep_route_count_kernel<8, 16, kDense>)
                           : go(ep_route_count_kernel<8, 32, kDense>);
    if (p.W <= 16)
        return p.k <= 8    ? go(ep_route_count_kernel<16, 8, kDense>)
               : p.k <= 16 ? go(ep_route_count_kernel<16, 16, kDense>)
                           : go(ep_route_count_kernel<16, 32, kDense>);
    return p.k <= 8    ? go(ep_route_count_kernel<32, 8, kDense>)
           : p.k <= 16 ? go(ep_route_count_kernel<32, 16, kDense>)
                       : go(ep_route_count_kernel<32, 32, kDense>);
}
}  // namespace

cudaError_t launch_route_count(const RouteParams& p, bool dense, cudaStream_t s) {
    const cudaError_t e = dense ? launch_route_count_as<true>(p, s) : launch_route_count_as<false>(p, s);
    return e != cudaSuccess ? e : cudaGetLastError();
}

size_t scatter_base_smem_bytes(int numTiles, int W) {
    return ((size_t)numTiles * (size_t)(W + 1) * sizeof(int) + 127) & ~(size_t)127;
}

size_t scatter_smem_bytes(int warps, int stages, int chunkStride) {
    const size_t head =
        ((size_t)warps * stages * (sizeof(uint64_t) + 2 * sizeof(int)) + 127) & ~(size_t)127;
    return head + (size_t)warps * stages * (size_t)chunkStride;
}

namespace {
template <typename F>
cudaError_t for_dense(bool dense, F&& f) {
    return dense ? f(ep_scatter_rows_kernel<1, true>) : f(ep_scatter_rows_kernel<1, false>);
}

// Raise a kernel's dynamic shared-memory limit to `bytes` (never lower it:
// plans and calls made earlier may rely on a larger limit).
template <typename K>
cudaError_t raise_smem(K kernel, size_t bytes) {
    cudaFuncAttributes fa;
    const cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    if ((size_t)fa.maxDynamicSharedSizeBytes >= bytes) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}
}  // namespace

cudaError_t scatter_set_smem(size_t bytes) {
    for (int d = 0; d < 2; ++d) {
        const cudaError_t e = for_dense(d != 0, [&](auto k) { return raise_smem(k, bytes); });
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t scatter_get_smem(int* bytes) {
    int lim = 1 << 30;
    for (int d = 0; d < 2; ++d) {
        cudaFuncAttributes fa;
        const cudaError_t e = for_dense(d != 0, [&](auto k) { return cudaFuncGetAttributes(&fa, k); });
        if (e != cudaSuccess) return e;
        lim = fa.maxDynamicSharedSizeBytes < lim ? fa.maxDynamicSharedSizeBytes : lim;
    }
    *bytes = lim;
    return cudaSuccess;
}

cudaError_t scatter_blocks_per_sm(int warps, size_t smem, int* out) {
    int lo = 1 << 30;
    for (int d = 0; d < 2; ++d) {
        int n = 0;
        const cudaError_t e = for_dense(d != 0, [&](auto k) {
            return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, warps * 32, smem);
        });
        if (e != cudaSuccess) return e;
        lo = n < lo ? n : lo;
    }
    *out = lo;
    return cudaSuccess;
}

namespace {
// The combine instance: 4 columns x 4 rows of 16-byte loads in flight per
// lane, 2 blocks of 256 threads per SM. A token's rows go in batches of 4, so
// a token with few destinations still keeps 16 loads in flight per lane.
// B200, against 2 columns x 8 rows: the 512-token workload (3.4 rows a token)
// 20.5 vs 24.8 us, skewed routing (2.7) 287 vs 304 us, main (5.3) 453.9 vs
// 453.7 us; 3 x 6 took 476 us at main; 2 x 4 at 4 or 3 blocks per SM and
// 1 x 8 at 4 were slower at main as well.
// kWide: the same tile in 32-byte loads, for large outputs (the host picks
// it). B200, main shape (W=8, h=7168, topk 8), 16- vs 32-byte loads: 4096
// tokens a rank 453.9 vs 441.7 us (fp32 rows 892.5 vs 868.2, skewed routing
// 287.4 vs 279.5), 2048 tokens 235.4 vs 233.9, but 1024 tokens 128.7 vs 136.1
// and the 512-token workload 20.6 vs 22.7: the wide loads pay only once the
// output is a few hundred MB.
template <class Elem, bool kWide = false>
constexpr auto combine_kernel = ep_combine_kernel<Elem, 4, 4, 2, kWide>;
}  // namespace

cudaError_t combine_blocks_per_sm(int warps, bool fp32, int* out) {
    return fp32 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, combine_kernel<CombineF32>, warps * 32, 0)
                : cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, combine_kernel<CombineBf16>, warps * 32, 0);
}

cudaError_t launch_scatter_rows(const ScatterParams& p, bool dense, int blocks, int warps, size_t smem,
                                cudaStream_t s) {
    cudaError_t e = for_dense(dense, [&](auto k) { return launch_pdl(k, blocks, warps * 32, smem, s, p); });
    return e != cudaSuccess ? e : cudaGetLastError();
}

namespace {
template <typename F>
cudaError_t for_world_fused(int W, int k, F&& f) {
    if (W <= 8)
        return k <= 8 ? f(ep_dispatch_fused_kernel<8, 8>) : k <= 16 ? f(ep_dispatch_fused_kernel<8, 16>)
                                                             : f(ep_dispatch_fused_kernel<8, 32>);
    if (W <= 16)
        return k <= 8 ? f(ep_dispatch_fused_kernel<16, 8>) : k <= 16 ? f(ep_dispatch_fused_kernel<16, 16>)
                                                              : f(ep_dispatch_fused_kernel<16, 32>);
    return k <= 8 ? f(ep_dispatch_fused_kernel<32, 8>) : k <= 16 ? f(ep_dispatch_fused_kernel<32, 16>)
                                                          : f(ep_dispatch_fused_kernel<32, 32>);
}
}  // namespace

cudaError_t fused_set_smem(int W, int topk, size_t bytes) {
    return for_world_fused(W, topk, [&](auto k) { return raise_smem(k, bytes); });
}

cudaError_t fused_blocks_per_sm(int W, int topk, size_t smem, int* out) {
    return for_world_fused(W, topk, [&](auto k) {
        return cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, k, kFusedWarps * 32, smem);
    });
}

cudaError_t launch_dispatch_fused(const ScatterParams& p, int blocks, size_t smem, cudaStream_t s) {
    cudaError_t e =
        for_world_fused(p.W, p.k, [&](auto k) { return launch_pdl(k, blocks, kFusedWarps * 32, smem, s, p); });
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_combine(const CombineParams& p, bool fp32, bool wide, int blocks, int warps, cudaStream_t s) {
    const cudaError_t e =
        fp32 ? (wide ? launch_pdl(combine_kernel<CombineF32, true>, blocks, warps * 32, 0, s, p)
                     : launch_pdl(combine_kernel<CombineF32>, blocks, warps * 32, 0, s, p))
             : (wide ? launch_pdl(combine_kernel<CombineBf16, true>, blocks, warps * 32, 0, s, p)
                     : launch_pdl(combine_kernel<CombineBf16>, blocks, warps * 32, 0, s, p));
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_comm_barrier_test(const BarrierTestParams& p, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.W);
    cfg.blockDim = dim3(32);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, ep_comm_barrier_test_kernel, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_comm_sync(const SyncParams& p, cudaStream_t s) {
    const cudaError_t e = launch_pdl(ep_comm_sync_kernel, 1, 32, 0, s, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_comm_push(const PushParams& p, int blocks, cudaStream_t s) {
    const cudaError_t e = launch_pdl(ep_comm_push_kernel, blocks, 256, 0, s, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace ep
