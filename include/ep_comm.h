/*
 * ep_comm.h -- expert parallelism across processes: one rank per process, each
 * on its own GPU (libep_b200.so).
 *
 * The same dispatch and combine as ep.h, with the W ranks real: rank r holds
 * only its own T token rows, and every rank's receive rows live in that
 * rank's GPU memory. The ranks share buffers through CUDA IPC handles, and the
 * kernels read and write the other ranks' buffers directly (over NVLink when
 * the GPUs are peers), in the way the design page's porting notes (§9) turn
 * symmetric-memory lookups into peer pointers: every rank maps every other
 * rank's shared buffers once, at connect time.
 *
 * One call, per rank:
 *   dispatch  1. route_count over this rank's T tokens: destinations, weight
 *                sums and this rank's count row (rows it sends to each rank);
 *             2. the count exchange: the count row goes into row `rank` of
 *                every rank's W x W count table (the aggregated, once per
 *                destination reservation of mori PR #599's follow-ups: a
 *                source's rows at destination pe start after those of the
 *                sources before it, so slots follow (source rank, token)
 *                ascending, exactly as on one GPU); barrier;
 *             3. the scatter pushes each token row and its meta record into
 *                the receive buffers of its destinations; barrier.
 *   combine   1. the push: every received row's expert output goes back to
 *                the landing rows of the rank it came from, at the offset the
 *                count table gives (the landing offsets that dispatch hands to
 *                the push combine); barrier;
 *             2. each rank folds its tokens' landing rows in ascending
 *                destination order, as ep_combine does.
 * The results are bit for bit those of ep_dispatch / ep_combine of the same
 * W-rank problem on one GPU: rank pe's receive rows, meta records and count
 * are destination pe's, and rank r's output rows are source r's.
 *
 * Barriers (EpSync):
 *   EP_SYNC_DEVICE  a one-warp kernel: each rank stores its barrier epoch (a
 *                   counter on the device, so replays of a captured graph
 *                   stay in step) into a flag of every rank, then waits until
 *                   all ranks' flags reach it. No host synchronisation: calls
 *                   can be captured in a CUDA graph. The wait gives up after
 *                   about a second and sets EP_DEVERR_TIMEOUT; the kernels
 *                   after it then touch no other rank, and the communicator
 *                   must be rebuilt. Every rank needs a GPU of its own:
 *                   ep_comm_connect refuses two ranks on one device.
 *   EP_SYNC_HOST    the host synchronises the stream and calls the caller's
 *                   barrier function (e.g. a torch.distributed barrier) at the
 *                   start of each call and between its steps. Ranks may share
 *                   a GPU. Not capturable. A rank that stops calling makes the
 *                   others' barrier function fail, and their call returns
 *                   EP_ERR_PEER before any kernel touches that rank's memory
 *                   (when the rank leaves between calls).
 */
#ifndef EP_COMM_B200_H
#define EP_COMM_B200_H

#include <stddef.h>
#include <stdint.h>

#include "ep.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum EpSync { EP_SYNC_DEVICE = 0, EP_SYNC_HOST = 1 } EpSync;

/* A rank's barrier function for EP_SYNC_HOST: returns 0 once every rank has
 * called it (the same number of times), nonzero when that cannot happen (a
 * rank left, a timeout). Called on the host thread that makes the call. */
typedef int (*EpHostBarrier)(void* ctx);

/* Another rank did not arrive (EP_SYNC_HOST): the call was abandoned. */
#define EP_ERR_PEER (-8)

/* Bytes of a rank's connection record (ep_comm_handle). */
#define EP_COMM_HANDLE_BYTES 256

typedef struct EpComm EpComm;

typedef struct EpCommInfo {
    int32_t rank;             /* this rank */
    int32_t worldSize;        /* W */
    int32_t sync;             /* EpSync */
    int32_t maxRecv;          /* receive rows of this rank */
    int32_t metaFields;       /* 3 + k */
    int32_t maxLanding;       /* landing rows of this rank: T * min(W, k) */
    int64_t rowBytes;         /* bytes of a dispatched row */
    int64_t combineRowBytes;  /* bytes of a y / out row */
    void* recvX;              /* device: this rank's receive rows [maxRecv][rowBytes] */
    int32_t* recvMeta;        /* device: their meta records [maxRecv][metaFields], as ep_dispatch's */
    int32_t* recvCount;       /* device: int32 [1], rows this rank received in the last dispatch */
    int64_t sharedBytes;      /* device memory other ranks map (receive rows, records, landing rows, tables) */
    int64_t localBytes;       /* device scratch of this rank only */
    int32_t scatterBlocks, scatterWarps, scatterStages, combineBlocks, combineWarps;
    int32_t device;           /* CUDA device of this rank */
} EpCommInfo;

/* Create rank `rank` of a W-rank communicator on the current CUDA device.
 * cfg is the shared configuration (every rank passes the same one):
 * worldSize = W ranks, maxTokPerRank = T token rows of each rank, maxRecv =
 * receive rows of each rank (>= W*T, 0 means W*T); the rest as in ep.h. sync:
 * EpSync; barrier/ctx: the host barrier (EP_SYNC_HOST only, else ignored).
 * Allocates this rank's shared and local device memory. Returns NULL on
 * failure (ep_last_error() says why). Test hook: EP_TEST_UNREACHABLE_BARRIER=1
 * makes every EP_SYNC_DEVICE barrier wait for an epoch no rank reaches. */
EpComm* ep_comm_create(const EpCfg* cfg, int32_t rank, int32_t sync, EpHostBarrier barrier, void* ctx);

/* This rank's connection record (EP_COMM_HANDLE_BYTES bytes into `out`): its
 * configuration, device and the IPC handle of its shared memory. Every rank
 * hands its record to every other rank (e.g. by an all-gather). */
int ep_comm_handle(const EpComm* comm, void* out);

/* Map every other rank's shared memory. `records`: the W connection records,
 * rank order, W * EP_COMM_HANDLE_BYTES bytes. Refuses records of another
 * configuration, and (EP_SYNC_DEVICE) two ranks on one GPU. Synchronous. */
int ep_comm_connect(EpComm* comm, const void* records);

int ep_comm_info(const EpComm* comm, EpCommInfo* info);

/* Dispatch this rank's tokens, enqueued on `stream`:
 *   x          dtype [T][h]    16-byte aligned
 *   topk_idx   int32 [T][k]    expert ids (< 0 masked)
 *   topk_w     float [T][k]    NULL allowed when useWeights == 0
 * Results in this rank's buffers (ep_comm_info: recvX, recvMeta, recvCount),
 * for the rows other ranks (and this one) sent here. Every rank must call it. */
int ep_comm_dispatch(EpComm* comm, const void* x, const int32_t* topk_idx, const float* topk_w,
                     void* stream);

/* Combine, enqueued on `stream`, with the routing of this rank's last
 * dispatch: y [maxRecv][hc] this rank's expert outputs in receive order
 * (16-byte aligned, rows < recvCount read; y may be recvX), out [T][hc] this
 * rank's output rows (every row written). hc and the types as ep_combine's.
 * Every rank must call it. */
int ep_comm_combine(EpComm* comm, const void* y, void* out, void* stream);

/* Synchronise the device; return and clear the error word (EP_DEVERR_*). */
int ep_comm_check_error(EpComm* comm);

/* Unmap the other ranks' memory and free this rank's. NULL is a no-op. No call
 * of any rank may still be running that uses this rank's memory. */
void ep_comm_destroy(EpComm* comm);

/* Self-test of the EP_SYNC_DEVICE barrier on the current GPU, without other
 * GPUs: W ranks (1..32) are the W blocks of one cooperative launch (so they
 * all run at once), each with its own flags, epoch and error word, meeting
 * `rounds` times. Before each barrier a rank writes a word; after it, it
 * reads every rank's word of that round, which must be there. Rank
 * `absentRank` (-1: none) stops arriving from round `absentFrom`; the others
 * then give up after about a second with EP_DEVERR_TIMEOUT. Per rank, into
 * host arrays of W (each may be NULL): barriers completed, error word, words
 * read too early. Synchronous; allocates and frees its own device memory.
 * Returns EP_OK or a negative code. */
int ep_comm_barrier_selftest(int32_t W, int32_t rounds, int32_t absentRank, int32_t absentFrom,
                             int32_t* roundsDone, int32_t* errors, int32_t* violations);

#ifdef __cplusplus
}
#endif

#endif /* EP_COMM_B200_H */
