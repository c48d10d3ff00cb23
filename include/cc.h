/* cc.h — collective primitives over N simulated ranks whose buffers all live in one
 * GPU's memory (B200, sm_100a). C ABI: plain pointers and sizes, no library types.
 *
 * Semantics follow the collective pages:
 *   lecture 09 "网络通信基础与集合通信 Collective 原语直觉" (§3 the eight primitives,
 *     §4 ring allreduce, §5 tree allreduce, §6 DDP / ZeRO / MoE dataflow, §7 experiments),
 *   "多节点训练集群网络优化实战" ch. 4 (§4.3.1 ring pseudocode, §4.3.2 double binary tree),
 *   "从零实现集合通信" (two-pass ring, per-rank byte table, gradient buckets).
 * Each rank's result is exactly what that rank would hold after the named schedule; a
 * floating-point reduction folds in the order the schedule implies:
 *   ring: chunk c (chunk rule below) is folded starting at rank c:
 *         ((x_c (+) x_{c+1}) (+) ...) (+) x_{c-1}   (indices mod N)
 *   tree: elements [0, ceil(count/2)) follow tree A, the rest tree B of the double
 *         binary tree; a node folds ((S_left (+) x_self) (+) S_right). Tree A is the
 *         in-order tree on positions 0..N-1 (1-based label q = position + 1, height
 *         h = ctz(q), left child q - 2^(h-1), right child q + 2^(j-1) for the largest
 *         j <= h with q + 2^(j-1) <= N, root = largest power of two <= N); tree B is its
 *         mirror (rank r at position N-1-r).
 *   chunk rule: q = count / N, r = count % N; chunk c has q + (c < r) elements and
 *         starts at c*q + min(c, r).
 * (+) is one IEEE binary32 operation rounded to nearest even (SUM add, PROD multiply,
 * MAX / MIN with -0 ordered below +0), or the wrapping int32 operation. bf16 inputs are
 * widened exactly to binary32 before the first operation. `scale` multiplies the final
 * result once (binary32); it must be 1 for int32. CC_SCALE_MEAN (any NaN) asks for the
 * average over the N ranks, the DDP step of lecture 09 §3.5 / §6.1 (AllReduce(SUM), then
 * divide by the card count): the library then multiplies by fl(1/N), computed in binary32
 * (exactly 1/N for N a power of two); for int32 it is CC_ERR_INVALID_ARG.
 *
 * Conventions for every call:
 *   - send / recv are HOST arrays of nranks DEVICE pointers (1 <= nranks <= 64), one per
 *     simulated rank; the caller owns all buffers; the library keeps no pointer after
 *     the call returns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     They return after enqueuing; only argument and launch errors are reported
 *     synchronously. A failed launch leaves the outputs undefined.
 *   - count == 0 is a no-op returning CC_OK.
 *   - Any alignment of 4-byte (2-byte for bf16) elements is accepted, with the same results
 *     on every path. 16-byte aligned buffers take 128-bit loads and stores; buffers that all
 *     sit the same whole number of elements past a 16-byte boundary take them after a short
 *     element-wise head; fp32 / int32 sums whose outputs sit at another offset than their
 *     sources take 128-bit loads and element stores; copies whose destinations share an
 *     offset that the source does not take 128-bit stores; everything else is element-wise.
 *   - In-place (recv[r] == send[r]) is allowed where stated; any other overlap between
 *     inputs and outputs is undefined.
 *   - Allowed (in, out) dtype pairs for reductions: (F32, F32), (BF16, F32), (I32, I32).
 */
#ifndef CC_H_
#define CC_H_

#include <math.h>
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CC_OK = 0,
  CC_ERR_INVALID_ARG = 1, /* bad pointer, size, rank, dtype pair, op or workspace */
  CC_ERR_UNSUPPORTED = 2, /* a valid combination this build does not implement */
  CC_ERR_CUDA = 3,        /* a CUDA runtime call failed (launch error, no device) */
  CC_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up (async status) */
} cc_status;

typedef enum { CC_F32 = 0, CC_BF16 = 1, CC_I32 = 2 } cc_dtype;
typedef enum { CC_SUM = 0, CC_MAX = 1, CC_MIN = 2, CC_PROD = 3 } cc_op;
typedef enum { CC_ALGO_RING = 0, CC_ALGO_TREE = 1 } cc_algo;

#define CC_MAX_RANKS 64

/* `scale` argument of the reductions meaning "the mean over the ranks": fl(1/N). */
#define CC_SCALE_MEAN (NAN)

#if defined(__GNUC__)
#define CC_API __attribute__((visibility("default")))
#else
#define CC_API
#endif

/* Human-readable name of a status code (static string). */
CC_API const char* cc_status_string(cc_status s);

/* Library version as major * 10000 + minor * 100 + patch. */
CC_API int cc_version(void);

/* Status of the device-side bounded waits (the bulk-copy pipeline of the data-movement
 * calls waits on shared-memory barriers with an iteration limit). Synchronizes `stream`,
 * then returns CC_OK, or CC_ERR_TIMEOUT if a wait gave up since the last reset (the outputs
 * of that call are then incomplete); `reset` != 0 clears the status. CC_ERR_CUDA if the
 * device cannot be read. A data-movement call whose tile load timed out (twice 2 s) leaves
 * with that load still in flight: its late write may land in shared memory the SM has
 * since given to other work, so results computed on that device after the timeout are
 * undefined as well; recreate the context before trusting it again. */
CC_API cc_status cc_async_status(int reset, void* stream);

/* Self-test of the device-side bounded waits: launches one thread that waits on a
 * shared-memory barrier nothing will ever complete; after timeout_us (1 .. 10^7) it gives
 * up and records CC_ERR_TIMEOUT in the status cc_async_status reads. Nothing faults or
 * traps; the context stays usable. For tests of the failure path only. */
CC_API cc_status cc_selftest_bounded_wait(unsigned timeout_us, void* stream);

/* The chunk rule (host only): chunk c of a count-element buffer over nranks ranks
 * starts at *start and has *len elements (lecture 09 §7.1 splits the tensor into N equal
 * chunks; for a count N does not divide, the first count % N chunks get one more). */
CC_API cc_status cc_chunk(size_t count, int nranks, int c, size_t* start, size_t* len);

/* AllReduce (lecture 09 §3.5; ring §4.3 and experiment 1 §7.1; tree §5.2 and the
 * multi-node page §4.3.2). Every rank r receives, in recv[r][0..count), the reduction of
 * send[0..N-1][0..count) folded in `algo`'s order, times `scale`.
 *   send[r]: count elements of in_t;  recv[r]: count elements of out_t.
 *   In place allowed (recv[r] == send[r] for every r, same dtype width).
 * Errors: CC_ERR_INVALID_ARG for null arrays/pointers, nranks outside [1, 64], a dtype
 * pair not listed above, op outside cc_op, scale != 1 for I32 (CC_SCALE_MEAN included). */
CC_API cc_status cc_allreduce(const void* const* send, void* const* recv, int nranks, size_t count,
                       cc_dtype in_t, cc_dtype out_t, cc_op op, cc_algo algo, float scale,
                       void* stream);

/* Stepped AllReduce: the same result as cc_allreduce, bit for bit, obtained by executing the
 * schedule's dependent steps one after another on the output buffers (ring: N-1
 * reduce-scatter steps then N-1 allgather steps, lecture 09 §4.3 and experiment 1 §7.1;
 * tree: the double binary tree reduced up one level per step and broadcast down one level
 * per step, lecture 09 §5.2, multi-node page §4.3.2). One cooperative launch with a grid
 * barrier between steps, so its time shows the schedule's latency (2(N-1) steps for the
 * ring against about 2 log2 N for the tree) next to its bandwidth.
 *   workspace: at least 256 bytes of device memory, 256-byte aligned, used for the grid
 *   barrier (cleared by the call, stream-ordered); calls that overlap on the GPU need
 *   separate workspaces.
 *   A barrier that does not complete within 2 s makes the kernel stop and record
 *   CC_ERR_TIMEOUT (see cc_async_status); outputs are then incomplete.
 * Other arguments, layouts and errors as cc_allreduce. */
CC_API cc_status cc_allreduce_stepped(const void* const* send, void* const* recv, int nranks, size_t count,
                                      cc_dtype in_t, cc_dtype out_t, cc_op op, cc_algo algo, float scale,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* Hierarchical AllReduce (lecture 09 §9.3 design question 1, appendix A Q4): the N ranks
 * form N / ranks_per_node nodes of ranks_per_node consecutive ranks. The result is what the
 * three-phase schedule leaves on every rank: a ring reduce-scatter inside every node, then
 * for every shard a ring allreduce across the nodes (ranks_per_node rings in parallel), then
 * a ring allgather inside every node. Element e of local chunk c (chunk rule over count with
 * ranks_per_node parts) and of sub-chunk j (chunk rule over chunk c with N / ranks_per_node
 * parts) folds x_{m,c} (+) x_{m,c+1} (+) ... inside each node m, and the node sums in node
 * order starting at node j; then `scale`. One fused pass (N·T in, N·T out). ranks_per_node
 * must divide nranks (else CC_ERR_INVALID_ARG); 1 or nranks give cc_allreduce's ring.
 * Other arguments as cc_allreduce. */
CC_API cc_status cc_allreduce_hierarchical(const void* const* send, void* const* recv, int nranks,
                                           int ranks_per_node, size_t count, cc_dtype in_t,
                                           cc_dtype out_t, cc_op op, float scale, void* stream);

/* Multi-ring AllReduce (lecture 09 §5.3: for large cross-node messages several rings run
 * side by side, one per NIC rail). The result is what this schedule leaves on every rank:
 * the count elements are cut into nrings contiguous parts (chunk rule with nrings parts),
 * and ring k runs the ring allreduce of cc_allreduce on part k (chunk rule with N parts
 * inside the part); even-numbered rings pass chunks to rank r + 1, odd-numbered rings run the
 * same schedule towards rank r - 1, so that with two or more rings both directions of every
 * link carry traffic. Chunk c of part k folds ((x_c (+) x_{c+1}) (+) ...) (+) x_{c-1} for even
 * k and ((x_c (+) x_{c-1}) (+) ...) (+) x_{c+1} for odd k; then `scale`. One fused pass (N·T
 * in, N·T out). nrings in [1, CC_MAX_RINGS] (else CC_ERR_INVALID_ARG); 1 gives
 * cc_allreduce's ring. Other arguments as cc_allreduce (in place allowed). */
#define CC_MAX_RINGS 64
CC_API cc_status cc_allreduce_multiring(const void* const* send, void* const* recv, int nranks, int nrings,
                                        size_t count, cc_dtype in_t, cc_dtype out_t, cc_op op, float scale,
                                        void* stream);

/* ReduceScatter (lecture 09 §3.6; the from-scratch page's reduce_scatter as the first
 * half of the ring). Rank c receives, in recv[c], chunk c (chunk rule) of the ring
 * reduction: q + (c < r) elements of out_t. `count` is the per-rank INPUT length.
 * algo must be CC_ALGO_RING (else CC_ERR_UNSUPPORTED). No in-place. */
CC_API cc_status cc_reduce_scatter(const void* const* send, void* const* recv, int nranks, size_t count,
                            cc_dtype in_t, cc_dtype out_t, cc_op op, cc_algo algo, float scale,
                            void* stream);

/* AllGather (lecture 09 §3.7; ring N-1 steps, the from-scratch page's table). Rank c
 * contributes send[c] = chunk c (chunk rule over `count`, the per-rank OUTPUT length);
 * every recv[r] receives all count elements. Bit copy; dtype only sets the width. */
CC_API cc_status cc_allgather(const void* const* send, void* const* recv, int nranks, size_t count,
                       cc_dtype dtype, void* stream);

/* Broadcast (lecture 09 §3.1; a log2(N) tree on the from-scratch page). Every recv[r]
 * receives the count elements at `src` (rank root's buffer). recv[root] may equal src
 * (then it is not written). Bit copy. */
CC_API cc_status cc_broadcast(const void* src, void* const* recv, int nranks, int root, size_t count,
                       cc_dtype dtype, void* stream);

/* Reduce to root (lecture 09 §3.4). recv_root receives the reduction of the N send
 * buffers over the binomial tree rooted at `root` (the broadcast tree run upward: node v
 * folds its own buffer, then each child's partial in the order it would send to them),
 * times `scale`. */
CC_API cc_status cc_reduce(const void* const* send, void* recv_root, int nranks, int root, size_t count,
                    cc_dtype in_t, cc_dtype out_t, cc_op op, float scale, void* stream);

/* Scatter (lecture 09 §3.2): recv[r] receives chunk r (chunk rule over `count`) of the
 * root buffer `src`. Gather (§3.3): recv_root receives the concatenation of send[r]
 * (chunk r of `count`) in rank order. Bit copies. */
CC_API cc_status cc_scatter(const void* src, void* const* recv, int nranks, int root, size_t count,
                     cc_dtype dtype, void* stream);
CC_API cc_status cc_gather(const void* const* send, void* recv_root, int nranks, int root, size_t count,
                    cc_dtype dtype, void* stream);

/* ---- MoE expert parallelism (lecture 09 §6.4, §3.8, experiment 4 §7.4) ---------------
 * Routing: expert_ids[r] ([tokens, topk] int32, device) receives, per token, the topk
 * largest of logits[r] ([tokens, experts_total] fp32, device), ties to the lower id,
 * larger first. topk in [1, 8], experts_total in [topk, 1024]. */
CC_API cc_status cc_route_topk(const float* const* logits, int32_t* const* expert_ids, int nranks,
                        int tokens, int experts_total, int topk, void* stream);

/* Workspace bytes cc_alltoallv needs (device memory, caller-allocated, 256-byte aligned). */
CC_API size_t cc_alltoallv_workspace_size(int nranks, int tokens, int topk, int experts_per_rank);

/* AllToAllv dispatch (direction 0) / combine (direction 1).
 * Expert e lives on rank e / experts_per_rank. Row (t, k) of source rank s is token t.
 * Dispatch: send[s] is [tokens, row_bytes]; recv[d] receives every row routed to rank d,
 *   as the concatenation over s = 0..N-1 of s's rows ordered by (local expert, t, k);
 *   at most recv_capacity_rows rows are written per rank (rows beyond it are dropped;
 *   cc_alltoallv_recv_counts tells the true counts).
 * Combine: send[d] is rank d's [rows, row_bytes] buffer in dispatch order; recv[s] is
 *   [tokens, topk, row_bytes] and receives each row back at slot [t][k].
 * An expert id outside [0, N * experts_per_rank) routes its row nowhere: dispatch sends it
 *   to no rank and combine leaves slot [t][k] of recv[s] as it was (so does a row that the
 *   capacity dropped).
 * Both directions rebuild the routing table from expert_ids in `workspace`.
 * row_bytes must be a positive multiple of 16. */
CC_API cc_status cc_alltoallv(const void* const* send, void* const* recv, int nranks, size_t row_bytes,
                       const int32_t* const* expert_ids, int tokens, int topk, int experts_per_rank,
                       size_t recv_capacity_rows, int direction, void* workspace,
                       size_t workspace_bytes, void* stream);

/* The two halves of cc_alltoallv, for a routing that serves more than one call (lecture 09
 * §6.4: the second AllToAll sends the experts' outputs back along the routes of the first, so
 * a dispatch and its combine share one routing).
 * cc_alltoallv_plan builds in `workspace` the routing tables cc_alltoallv builds at every call
 * (per-source tile counts and prefixes, per-row ranks, bases, receive counts) from expert_ids;
 * cc_alltoallv_run does only the row copy of cc_alltoallv, in either direction, reading the
 * tables that the last plan (or the last cc_alltoallv) left in `workspace`. A run gives exactly
 * cc_alltoallv's result as long as expert_ids, tokens, topk, experts_per_rank and nranks are
 * those of that plan and nothing else wrote the workspace in between; after expert_ids change,
 * plan again. Arguments, layouts, workspace rules and errors as cc_alltoallv (plan takes no
 * row buffers). cc_alltoallv_recv_counts reads the counts of the last plan. */
CC_API cc_status cc_alltoallv_plan(const int32_t* const* expert_ids, int nranks, int tokens, int topk,
                                   int experts_per_rank, void* workspace, size_t workspace_bytes, void* stream);
CC_API cc_status cc_alltoallv_run(const void* const* send, void* const* recv, int nranks, size_t row_bytes,
                                  const int32_t* const* expert_ids, int tokens, int topk, int experts_per_rank,
                                  size_t recv_capacity_rows, int direction, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Copies the per-destination received row counts of the last cc_alltoallv or
 * cc_alltoallv_plan that used `workspace` into recv_rows[0..nranks) (host or device memory),
 * stream-ordered. */
CC_API cc_status cc_alltoallv_recv_counts(const void* workspace, int nranks, int32_t* recv_rows,
                                   void* stream);

/* cc_alltoallv without a workspace, for callers that cannot allocate device memory
 * (a plugin or custom-operator host that hands over only inputs and outputs, or a runtime
 * that keeps all device memory in its own pool). The collective pages have no counterpart;
 * this is a deployment variant of cc_alltoallv with the same arguments and results.
 *   Scratch: a fixed 1 MiB array inside the library's device memory, one per GPU, held by
 *   every GPU that loads the library until the process exits. Shapes whose routing scratch
 *   (cc_alltoallv_workspace_size) exceeds 1 MiB are rejected with CC_ERR_INVALID_ARG
 *   (N = 8, 8192 tokens, top-2, 8 experts per rank needs 644 KiB).
 *   Set-up: the first call on a device looks up the array's device address with that
 *   device current; make that first call before any stream capture.
 *   Sharing: every call on a device uses the same array and leaves its tables there; each
 *   call rewrites every entry it reads, so nothing needs clearing, but calls that overlap
 *   on the GPU (other streams, other threads) race: serialize them.
 *   recv_rows: NULL, or nranks int32 (device or pinned host memory) that receive the
 *   per-destination row counts, stream-ordered.
 *   Allocates nothing: no cudaMalloc, no cudaFree. */
CC_API cc_status cc_alltoallv_noalloc(const void* const* send, void* const* recv, int nranks,
                                      size_t row_bytes, const int32_t* const* expert_ids, int tokens,
                                      int topk, int experts_per_rank, size_t recv_capacity_rows,
                                      int direction, int32_t* recv_rows, void* stream);

/* ---- DDP gradient buckets (lecture 09 §6.1; the from-scratch page's bucketing) --------
 * Bucket assignment (host only): tensors are taken in reverse order of their index
 * (the order backward produces them), never split; a new bucket starts when the next
 * tensor would push a non-empty bucket past cap_bytes. Outputs: order[0..ntensors) =
 * tensor ids in bucket order, bucket_start[0..nbuckets] = offsets into `order`,
 * *nbuckets. bucket_start must have room for ntensors + 1 entries. */
CC_API cc_status cc_bucket_assign(const size_t* numels, int ntensors, size_t elem_bytes, size_t cap_bytes,
                           int32_t* order, int32_t* bucket_start, int32_t* nbuckets);

/* Flatten: bucket[off_i .. off_i + numels[i]) = tensors[i], off_i = prefix sum, for the
 * ntensors tensors in the given order. Unflatten is the inverse. Bit copies. */
CC_API cc_status cc_bucket_flatten(const void* const* tensors, const size_t* numels, int ntensors,
                            void* bucket, cc_dtype dtype, void* stream);
CC_API cc_status cc_bucket_unflatten(const void* bucket, void* const* tensors, const size_t* numels,
                              int ntensors, cc_dtype dtype, void* stream);

/* Fused DDP step: for every bucket of cc_bucket_assign(numels, 4, cap_bytes), the result
 * of flatten -> allreduce(algo, SUM, scale) -> unflatten, computed in one pass without
 * the flat buffers: out[r * ntensors + i] receives tensor i of rank r.
 *   grads / out: host arrays of nranks * ntensors device pointers (rank-major,
 *   registration order); F32; in place allowed (out[j] == grads[j] for every j).
 * The pointer and bucket tables travel as kernel parameters (no workspace); a tensor
 * list longer than one launch can carry is split into several launches. */
CC_API cc_status cc_bucket_allreduce(const void* const* grads, void* const* out, int nranks, int ntensors,
                              const size_t* numels, size_t cap_bytes, cc_algo algo, float scale,
                              void* stream);

/* Buckets [first_bucket, first_bucket + nbuckets) of the assignment cc_bucket_assign makes
 * for the whole tensor list, with the same results as cc_bucket_allreduce for their tensors
 * (other tensors are not touched). This is how a training step overlaps the allreduce with
 * backward (lecture 09 §6.1 bucket overlap; the from-scratch page's bucket-ready hooks):
 * buckets come in the order backward produces gradients, so bucket b can be launched on a
 * side stream as soon as its last gradient is written (cudaStreamWaitEvent on an event
 * recorded after it). CC_ERR_INVALID_ARG if the range exceeds the bucket count. */
CC_API cc_status cc_bucket_allreduce_buckets(const void* const* grads, void* const* out, int nranks,
                                             int ntensors, const size_t* numels, size_t cap_bytes,
                                             int first_bucket, int nbuckets, cc_algo algo, float scale,
                                             void* stream);

/* The same fused DDP step for gradients that live in host memory: every host_grads[j] is
 * copied to dev_grads[j] (host -> device), the fused allreduce runs on the device copies,
 * and every dev_out[j] is copied back to host_out[j] (device -> host). The work is cut in
 * registration order into slices (at most 2^20 elements per rank) grouped into stages, and the
 * copies in, the kernels and the copies out of consecutive stages overlap on two
 * library-owned streams (created once per device) and `stream`; a slice keeps its bucket
 * offset, so the results equal cc_bucket_allreduce's. From the caller's view the call is
 * ordered on `stream` (it starts after earlier work on `stream`; later work on `stream`
 * sees the host outputs written). The caller owns the device staging buffers (dev_grads
 * may equal dev_out); host buffers must be pinned for the copies to overlap.
 * packed != 0 promises that, for each rank and each of the four tables, the rank's
 * tensors lie in one allocation (for instance views of one flat gradient buffer per
 * rank): a stage's copies that are then contiguous on both sides are merged into one
 * transfer. With packed == 0 a copy never spans two tensors (two allocations may happen
 * to be adjacent, and one copy may not cross from one into the other). Layouts as
 * cc_bucket_allreduce. */
CC_API cc_status cc_bucket_allreduce_host(const void* const* host_grads, void* const* host_out,
                                          void* const* dev_grads, void* const* dev_out, int nranks,
                                          int ntensors, const size_t* numels, size_t cap_bytes,
                                          cc_algo algo, float scale, int packed, void* stream);

/* ---- One rank's slice, for ranks in separate processes (one per GPU) ----------------------
 * The same schedules with the N ranks' buffers on N GPUs, one process each: every rank's
 * buffers are mapped into each process (cc_ipc_open of the other processes' exports, or
 * plain device pointers for this process's own), and rank `rank` does only its own share
 * of the single-GPU call, loading peer inputs and storing into peer outputs directly over
 * NVLink with ordinary loads and stores (no bulk or multicast copy touches peer memory).
 * This is the ring's ownership split (lecture 09 §4.2-4.3: after the reduce-scatter, rank
 * c holds the full sum of chunk c; the allgather then hands that chunk to everyone) run as
 * one pass: rank c folds chunk c (chunk rule) from all N inputs and writes it to all N
 * outputs, so the whole exchange is one fold per element and every byte crosses NVLink
 * once each way.
 * The caller orders the ranks: every input written (and every output no longer read)
 * before any rank starts, and no output read before every rank has finished, e.g. a
 * stream synchronisation plus a process-group barrier on both sides. Once all N ranks
 * have made the call, the outputs hold exactly what the single-process call writes, bit
 * for bit. `rank` outside [0, nranks) is CC_ERR_INVALID_ARG; other arguments, layouts and
 * errors as the single-process call. */

/* Allreduce: rank `rank` folds the elements of chunk `rank` (in the ring order of the
 * chunk for CC_ALGO_RING, in the tree order of the half each element falls in for
 * CC_ALGO_TREE) and writes them, scaled, into all N recv buffers. In-place allowed. */
CC_API cc_status cc_allreduce_slice(const void* const* send, void* const* recv, int nranks, int rank,
                                    size_t count, cc_dtype in_t, cc_dtype out_t, cc_op op, cc_algo algo,
                                    float scale, void* stream);

/* Reduce-scatter (ring order): rank `rank` folds chunk `rank` of all N send buffers into
 * its own shard recv_shard (chunk `rank`'s length; may be NULL when that is 0). */
CC_API cc_status cc_reduce_scatter_slice(const void* const* send, void* recv_shard, int nranks, int rank,
                                         size_t count, cc_dtype in_t, cc_dtype out_t, cc_op op, float scale,
                                         void* stream);

/* Allgather: rank `rank` copies its shard (chunk `rank` of the count) into that chunk of
 * all N recv buffers. */
CC_API cc_status cc_allgather_slice(const void* send_shard, void* const* recv, int nranks, int rank,
                                    size_t count, cc_dtype dtype, void* stream);

/* CUDA IPC for the slice calls. cc_ipc_export writes an opaque handle (cc_ipc_handle_bytes()
 * bytes, caller-owned) for the device allocation that holds dev_ptr, and the byte offset of
 * dev_ptr inside it; any other process on the node passes both to cc_ipc_open to get a
 * pointer to the same bytes (peer access is enabled on first use). Opening the same
 * allocation several times in a process maps it once (reference-counted); cc_ipc_close
 * undoes one cc_ipc_open. The exporting process must keep the allocation alive until every
 * importer has closed it. Opening a handle in the process that exported it is
 * CC_ERR_CUDA (use the local pointer). */
CC_API size_t cc_ipc_handle_bytes(void);
CC_API cc_status cc_ipc_export(const void* dev_ptr, void* handle, size_t* offset);
CC_API cc_status cc_ipc_open(const void* handle, size_t offset, void** dev_ptr);
CC_API cc_status cc_ipc_close(void* dev_ptr);

#ifdef __cplusplus
}
#endif

#endif /* CC_H_ */
