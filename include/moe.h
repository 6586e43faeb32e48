/*
 * moe.h -- C ABI of libmoe_b200.so: the forward and backward passes of one
 * deterministic Mixture-of-Experts layer on one B200 (sm_100a).
 *
 * The layer has four steps:
 *   1. top-k routing from router logits;
 *   2. the pull-dispatch schedule table Phi, built on the device as a
 *      single-pass counting sort;
 *   3. a pull gather of the tokens into contiguous per-expert buffers and a
 *      grouped SwiGLU expert FFN (bf16 operands, fp32 accumulation);
 *   4. a gate-weighted combine back to token order in a fixed floating-point
 *      order, so identical inputs give bitwise-identical outputs.
 * The backward pass (training) reuses the forward's Phi for both of its
 * exchanges (see the "Backward" section at the end of this header).
 *
 * Sources (page title, section):
 *   "Mixture-of-Kittens: A MoE Megakernel for GB300 NVL72" (MoK notes),
 *     section 2 "Push vs. Pull" (two-column pull table; on-device schedule
 *     generation with counts T, M, offsets S and the stable cross-rank
 *     position p), section 3 "The Goldilocks Minibatch Size T",
 *     section 5 "Megakernel Fusion" (SwiGLU expert GEMMs).
 *   "Scan once, scatter once", section "The fix is a counting sort" (count,
 *     prefix, pad to 256 rows, scatter once).
 *   "Beyond Peak TFLOPs", sections 2.A and 2.B (pull dispatch / push combine,
 *     no dynamic allocation or host round trips) and its opening (bitwise
 *     reproducible outputs from a fixed floating-point order).
 *
 * Expert-parallel peers are logical partitions of one GPU's memory: peer r
 * owns tokens r*N .. r*N+N-1 of every [P*N, ...] token array.
 *
 * Conventions for every entry point:
 *   - All pointers are DEVICE pointers unless the name ends in _host.
 *     bf16 tensors are passed as uint16_t bit patterns. All arrays are dense,
 *     row-major, and must be 16-byte aligned (256-byte alignment recommended);
 *     the FFN outputs h, ab and y, the weight gradients and every workspace
 *     must be 32-byte aligned.
 *   - The caller owns and allocates every buffer; the library never allocates
 *     device memory and never synchronises with the host. Work is enqueued on
 *     `stream` (a cudaStream_t; NULL = the legacy default stream) and runs
 *     asynchronously; results are valid once the stream has been synchronised.
 *   - Errors found from the arguments alone are returned synchronously as a
 *     moe_status_t, before anything is enqueued. Errors that depend on data
 *     (an expert id outside [0,E), an inconsistent schedule, a device wait
 *     that timed out) are OR-ed as MOE_DEV_* flags into *dev_status, which
 *     the caller zeroes beforehand and reads after synchronising. Kernels never
 *     trap: on bad data they skip the offending element and raise the flag.
 *   - Calls that share buffers must not overlap on the GPU.
 *   - Shape limits: 1 <= P <= 64; 0 <= N; 1 <= E <= 1024; 1 <= k <= min(E, 16);
 *     P*N*k and the padded row count below 2^31. The expert FFN and the layer
 *     additionally need H % 256 == 0, I % 128 == 0, pad % 128 == 0.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Problem shape. P peers x N tokens each, E experts, top-k routing, hidden
 * size H, expert intermediate size I, expert segment padding `pad` rows
 * (256 in the pages' scheduler). */
typedef struct moe_shape {
  int32_t P, N, E, k, H, I, pad;
} moe_shape_t;

typedef int moe_status_t;
enum {
  MOE_OK = 0,
  MOE_INVALID_ARG = 1,          /* null pointer, negative size, misaligned buffer */
  MOE_UNSUPPORTED_SHAPE = 2,    /* shape outside the limits above */
  MOE_WORKSPACE_TOO_SMALL = 3,
  MOE_CUDA_ERROR = 4,           /* a CUDA runtime call failed (e.g. no device) */
  MOE_DEVICE_TIMEOUT = 5,       /* host view of MOE_DEV_TIMEOUT */
  MOE_BAD_EXPERT_ID = 6,        /* host view of MOE_DEV_BAD_EXPERT_ID */
  MOE_BAD_SCHEDULE = 7          /* host view of MOE_DEV_BAD_SCHEDULE */
};

/* Flags OR-ed into *dev_status by kernels. */
#define MOE_DEV_BAD_EXPERT_ID 0x1  /* an id outside [0,E): that route is dropped */
#define MOE_DEV_TIMEOUT       0x2  /* a bounded device wait gave up (~1 s) */
#define MOE_DEV_BAD_SCHEDULE  0x4  /* offsets/Phi/route_row out of range: element skipped */

/* Human-readable name of a status code (static string). */
const char* moe_status_string(moe_status_t s);

/* Status code for a set of MOE_DEV_* flags (the most severe one; MOE_OK if 0). */
moe_status_t moe_status_from_device_flags(int32_t flags);

/* Upper bound on the rows of the padded, expert-sorted layout:
 * P*N*k + E*(pad-1), rounded up to a multiple of pad (and of 256).
 * Phi, the gathered buffer xg, h and y are sized with it. -1 on a bad shape. */
int64_t moe_rows_max(const moe_shape_t* shape);

/* Bytes of scratch `ws` that moe_schedule needs for `shape`. */
size_t moe_schedule_workspace_bytes(const moe_shape_t* shape);

/* Bytes of scratch `ws` that moe_layer_forward needs (ids, gates, Phi,
 * offsets, counts, route_row, the schedule's scratch, the GEMMs' tile counter
 * and landing flags, xg, h and y). */
size_t moe_layer_workspace_bytes(const moe_shape_t* shape);

/* Bytes of scratch for moe_layer_forward_host: the above plus device copies
 * of the logits, the activations and the output. */
size_t moe_layer_host_workspace_bytes(const moe_shape_t* shape);

/* Step 1 -- top-k routing ("routing tensor" of MoK notes section 2; gates as
 * the softmax over the chosen logits).
 * logits: fp32 [P*N, E]. For each token the k largest logits are chosen in
 * descending order, ties to the lower expert id; ids: int32 [P*N, k] (slot j
 * = j-th largest); gates: fp32 [P*N, k], gates[t,j] = exp(l_j - l_0) /
 * sum_j' exp(l_j' - l_0). Logits must be finite or -inf, with at least one
 * finite logit per token. */
moe_status_t moe_route_topk(const float* logits, int32_t* ids, float* gates,
                            const moe_shape_t* shape, void* stream);

/* Step 2 -- the pull-dispatch schedule Phi ("Scan once, scatter once", the
 * four stages of "The fix is a counting sort"; placement of MoK notes
 * section 2).
 * ids: int32 [P, N, k]; route (r, q), q = i*k + j, is slot j of token i of
 * peer r. With M[l,r] = routes of peer r to expert l, T[l] = sum_r M[l,r],
 * Tp[l] = ceil(T[l]/pad)*pad and S the exclusive prefix sum of Tp:
 *   offsets: int32 [E+1] = S (offsets[E] = rows in use);
 *   counts:  int32 [E, P] = M;
 *   phi:     int32 [moe_rows_max, 2]; row S[l]+p holds (src_rank, src_idx) =
 *            (r, i) of the route whose stable rank within (l, r) is o (routes
 *            of one peer in ascending q), where
 *            p = sum_{r'} min(M[l,r'], o) + |{r' < r : M[l,r'] > o}|;
 *            rows S[l]+T[l] .. S[l+1]-1 hold (-1,-1); rows >= offsets[E] are
 *            not written;
 *   route_row: int32 [P, N, k] = the Phi row of each route.
 * ws: scratch of moe_schedule_workspace_bytes (contents irrelevant on entry).
 * An id outside [0,E) raises MOE_DEV_BAD_EXPERT_ID, is not placed, and its
 * route_row is -1. Each route is read twice (count, scatter). */
moe_status_t moe_schedule(const int32_t* ids, int32_t* phi, int32_t* offsets, int32_t* counts,
                          int32_t* route_row, void* ws, size_t ws_bytes, int32_t* dev_status,
                          const moe_shape_t* shape, void* stream);

/* moe_schedule without a caller-provided scratch buffer. The source pages have
 * no counterpart: this entry point exists for callers that cannot allocate
 * device memory for `ws` -- for instance a plugin that a host application
 * calls with only its input and output buffers, or a serving loop that bans
 * cudaMalloc on its hot path because an allocation can synchronise the device.
 * Arguments, outputs and device-status behaviour are those of moe_schedule.
 * The scratch is a fixed 4 MiB device array inside the library (1,048,576
 * int32 words; every GPU that loads the library holds it until the process
 * exits); shapes needing more, i.e. P * ceil(N*k/2048) * E > 1,048,576, are
 * rejected with MOE_WORKSPACE_TOO_SMALL before anything is enqueued. The
 * first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture. Under lazy module loading (the CUDA default) that first call may
 * also load the library's device code, the 4 MiB array with it; later calls
 * allocate nothing. The address is kept for the life of the process: after a
 * cudaDeviceReset the kept address is stale, so do not call this entry point
 * on that device again in the same process. All calls share the one array
 * and it keeps the last call's contents (the kernels overwrite every word
 * they read), so calls that overlap on the GPU -- e.g. on two streams at
 * once -- race and must be serialised by the caller. Calls no cudaMalloc,
 * cudaFree or other allocating routine. */
moe_status_t moe_schedule_static_ws(const int32_t* ids, int32_t* phi, int32_t* offsets,
                                    int32_t* counts, int32_t* route_row, int32_t* dev_status,
                                    const moe_shape_t* shape, void* stream);

/* Step 3a -- pull dispatch ("Beyond Peak TFLOPs" 2.A, MoK notes section 2:
 * tokens land zero-copy in contiguous per-expert buffers).
 * x: bf16 [P*N, H]; xg: bf16 [moe_rows_max, H]. For row < offsets[E]:
 * xg[row] = x[src_rank*N + src_idx] with (src_rank, src_idx) = phi[row], and
 * padding rows (src_rank < 0) are zero. Rows >= offsets[E] are not written.
 * An out-of-range Phi entry raises MOE_DEV_BAD_SCHEDULE and zeroes the row. */
moe_status_t moe_dispatch(const uint16_t* x, const int32_t* phi, const int32_t* offsets,
                          uint16_t* xg, int32_t* dev_status, const moe_shape_t* shape,
                          void* stream);

/* Step 3b -- grouped SwiGLU expert FFN (MoK notes section 5), a persistent
 * tcgen05 grouped GEMM pair with bf16 operands and fp32 accumulation.
 * W1 (gate), W3 (up): bf16 [E, H, I]; W2 (down): bf16 [E, I, H].
 * For every row in expert l's segment [offsets[l], offsets[l+1]):
 *   h[row] = bf16_rne( silu(xg[row].W1[l]) * (xg[row].W3[l]) ),  h: bf16 [moe_rows_max, I]
 *   y[row] = h[row].W2[l] (fp32),                                 y: fp32 [moe_rows_max, H]
 * counts (int32 [E,P], may be NULL): when given, tiles that hold only
 * padding rows are skipped and their h/y rows are left unwritten, and y is
 * not written for 32-row blocks past the last route of their expert; rows
 * that carry routes are always written. Each output element is computed by one
 * CTA (pair) with a fixed K order: the result is bitwise deterministic.
 * Tile counter: the GEMM kernels take their tiles from a counter of two
 * int32 words that the last CTA of each launch puts back to zero. The GEMM
 * entry points without a workspace (this one, moe_expert_ffn_gather,
 * moe_expert_ffn_train, _dgrad, _wgrad, _mxfp8) take the next of 256 such
 * counters per device, round robin; nothing is written to a counter when a
 * launch is enqueued, so FFN calls on different streams may run at the same
 * time. Two launches share a counter only if both run at the same moment
 * with 255 other such launches enqueued between them, or if one captured
 * graph holding them is replayed on two streams at once: neither is allowed.
 * The layer entry points keep their counter in `ws` instead.
 * offsets must be non-decreasing multiples of 128 with offsets[E] <=
 * moe_rows_max (else MOE_DEV_BAD_SCHEDULE, nothing written). */
moe_status_t moe_expert_ffn(const uint16_t* xg, const uint16_t* W1, const uint16_t* W3,
                            const uint16_t* W2, const int32_t* offsets, const int32_t* counts,
                            uint16_t* h, float* y, int32_t* dev_status,
                            const moe_shape_t* shape, void* stream);

/* Steps 3a + 3b fused -- the pull dispatch lands the tokens directly in the
 * FFN's operand tiles ("Mixture-of-Kittens" notes section 2, zero-copy direct
 * landing; "Beyond Peak TFLOPs" 2.A): GEMM1 reads row `row` of its A operand
 * as x[src_rank*N + src_idx] with (src_rank, src_idx) = phi[row] (zeros for
 * padding rows) with 16-byte asynchronous copies, so no gathered buffer
 * exists.
 * x: bf16 [P*N, H]; phi: int32 [moe_rows_max, 2] as written by moe_schedule;
 * everything else as moe_expert_ffn, whose h and y it reproduces bit for bit.
 * An out-of-range Phi entry raises MOE_DEV_BAD_SCHEDULE and reads as zeros.
 * It needs no [moe_rows_max, H] gathered buffer, but on B200 its GEMM1 runs
 * about 2.6x slower than moe_dispatch + moe_expert_ffn (each gathered A tile
 * is re-read for every output column block, and row gathers deliver fewer
 * bytes per clock than the tensor cores consume), so moe_layer_forward uses
 * the latter. */
moe_status_t moe_expert_ffn_gather(const uint16_t* x, const int32_t* phi, const uint16_t* W1,
                                   const uint16_t* W3, const uint16_t* W2, const int32_t* offsets,
                                   const int32_t* counts, uint16_t* h, float* y,
                                   int32_t* dev_status, const moe_shape_t* shape, void* stream);

/* Step 4 -- push combine in a fixed floating-point order ("Scan once, scatter
 * once" opening and "Beyond Peak TFLOPs" opening: bitwise-reproducible outputs).
 * out[t] = bf16_rne(acc) with acc = 0.0f; acc = fmaf(gates[t,j], y[route_row[t,j]], acc)
 * for j = 0..k-1 in ascending order. out: bf16 [P*N, H]. A route_row outside
 * [0, moe_rows_max) contributes nothing and raises MOE_DEV_BAD_SCHEDULE. */
moe_status_t moe_combine(const float* y, const int32_t* route_row, const float* gates,
                         uint16_t* out, int32_t* dev_status, const moe_shape_t* shape,
                         void* stream);

/* Steps 1-4 in one call, all enqueued on `stream` with no host round trip.
 * When pad % 256 == 0 (CTA-pair tiles) the pull dispatch runs inside the
 * FFN's first GEMM ("Mixture-of-Kittens" notes section 2, tokens landing in
 * the buffers the experts read; "Beyond Peak TFLOPs" section 3, one kernel
 * overlapping data movement with the MMAs): a spare warp of every CTA copies
 * 128-row blocks of x into the gathered buffer through Phi while the tensor
 * cores work on blocks already landed; the result is bit for bit that of
 * moe_dispatch + moe_expert_ffn.
 * minibatch_tokens: transfer slice T in tokens per peer (MoK notes section 3);
 * 0 or >= N = one slice. Slice s covers tokens [s*T, (s+1)*T) of every peer and
 * runs schedule -> dispatch -> FFN -> combine on them; routing runs once over
 * all tokens. Every output row is computed with the same arithmetic whatever
 * the slicing, so out is bitwise identical for every T.
 * ws: scratch of moe_layer_workspace_bytes. stage_events: NULL, or an array of
 * 7 cudaEvent_t recorded (single-slice runs only) before routing, schedule,
 * dispatch, FFN GEMM1, FFN GEMM2, combine, and after combine. */
moe_status_t moe_layer_forward(const float* logits, const uint16_t* x, const uint16_t* W1,
                               const uint16_t* W3, const uint16_t* W2, uint16_t* out,
                               int32_t minibatch_tokens, void* ws, size_t ws_bytes,
                               int32_t* dev_status, const moe_shape_t* shape, void* stream,
                               void* const* stage_events);

/* moe_layer_forward with HOST inputs and output: logits_host fp32 [P*N, E],
 * x_host bf16 [P*N, H] and out_host bf16 [P*N, H] live in host memory (pinned
 * memory makes the copies asynchronous); the weights, ws (of
 * moe_layer_host_workspace_bytes) and dev_status are device memory.
 * Copies overlap compute in two ways:
 *   - across calls: consecutive calls alternate between two device copies of
 *     the inputs inside ws, so the host-to-device copy of a call starts as
 *     soon as the call is made and runs while the previous call computes
 *     (it waits only for the call before that to finish reading the same
 *     copies). The host inputs must therefore hold their values when the
 *     call is made, not only when earlier work on `stream` has finished.
 *   - within a call, at the transfer slice `minibatch_tokens` (MoK notes
 *     section 3; "Beyond Peak TFLOPs" section 1: chunk k moves while chunk
 *     k-1 computes): slice s+1's rows are copied in and slice s-1's outputs
 *     copied out while slice s computes. 0 = one slice.
 * The copies run on two internal streams per device (host-to-device,
 * device-to-host) with a few events, created on the first call on that
 * device and kept until exit; `stream` waits for every copy of the call, so
 * out_host is valid once `stream` has been synchronised. Calls from several
 * host threads are serialised. */
moe_status_t moe_layer_forward_host(const float* logits_host, const uint16_t* x_host,
                                    const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                                    uint16_t* out_host, int32_t minibatch_tokens, void* ws,
                                    size_t ws_bytes, int32_t* dev_status,
                                    const moe_shape_t* shape, void* stream);

/* moe_layer_forward_host whose copy of the output to the host runs off
 * `stream`: `stream` orders the input copies and the compute, and the copy of
 * out_host completes when out_ready (a cudaEvent_t the caller created, ideally
 * with cudaEventDisableTiming) completes; `stream` does not wait for it. So
 * consecutive calls compute back to back while each call's output travels to
 * the host (the device keeps two output copies in ws and call i+2 reuses call
 * i's only after it has been copied out). out_host holds the output once
 * out_ready has completed; the copies out of all host-buffer calls on a
 * device run in call order on one internal stream, so a later call may be
 * handed the same out_host. Everything else as moe_layer_forward_host (same
 * workspace size). */
moe_status_t moe_layer_forward_host_async(const float* logits_host, const uint16_t* x_host,
                                          const uint16_t* W1, const uint16_t* W3,
                                          const uint16_t* W2, uint16_t* out_host,
                                          int32_t minibatch_tokens, void* ws, size_t ws_bytes,
                                          int32_t* dev_status, const moe_shape_t* shape,
                                          void* stream, void* out_ready);

/* ------------------------------------------------------------------------
 * Backward (training).
 *
 * "Mixture-of-Kittens: A MoE Megakernel for GB300 NVL72": one schedule table
 * serves all four forward and backward phases (overview), the backward being
 * pull-reverse-combine and push-reverse-dispatch (section 2); weight
 * gradients are deferred until every activation gradient is done and
 * accumulated over the token dimension in one pass for bitwise
 * reproducibility (overview, backward execution step); the router gradient
 * is the inner product of the SwiGLU activations and the down-projection
 * dgrads, so the down projection's output is never kept (section 5,
 * SonicMoE gradients); forward activations are kept, not recomputed.
 *
 * For route (t, j) with expert e, gate g = gates[t,j] and row = route_row[t,j]
 * (the forward saved a = xg.W1[e], b = xg.W3[e] as bf16 and h as bf16):
 *   dhu   = dout[t] . W2[e]^T                             (fp32)
 *   dgate = sum_i h[i] * dhu[i]
 *   dh    = g * dhu;  s = 1 / (1 + exp(-a))
 *   da    = bf16(dh * b * s * (1 + a (1 - s))),  db = bf16(dh * a * s),
 *   hg    = bf16(g * h)
 *   dxg   = da . W1[e]^T + db . W3[e]^T                   (fp32)
 *   dx[t] = bf16(sum_j dxg[route_row[t,j]])               (ascending j, from 0)
 *   dlogits[t, ids[t,j]] = g_j (dgate_j - sum_j' g_j' dgate_j'), 0 elsewhere
 *   dW1[e] = sum over e's rows of xg^T da, dW3[e] = xg^T db, dW2[e] = hg^T dout
 *                                                         (fp32, one pass)
 * Every output element is produced by one thread or one CTA pair in a fixed
 * order (no atomics, no split-K): the gradients are bitwise reproducible.
 * Shape limits in addition to the FFN's: I % 256 == 0 and pad % 256 == 0
 * (every GEMM runs 256 x 256 tiles on CTA pairs). Weight gradients are
 * written whole: an expert that received no route gets zeros.
 * ------------------------------------------------------------------------ */

/* Bytes of the workspace of moe_layer_forward_train / moe_layer_backward
 * (0 if the shape is unsupported): the forward's buffers plus the saved
 * pre-activations and the backward's buffers (about rows * (9H + 12I) bytes). */
size_t moe_train_workspace_bytes(const moe_shape_t* shape);

/* moe_expert_ffn that also keeps the pre-activations for the backward:
 * ab: bf16 [moe_rows_max, 2I], ab[row] = [bf16(a) | bf16(b)] with a, b the
 * fp32 accumulators of GEMM1 (written for the rows moe_expert_ffn writes h). */
moe_status_t moe_expert_ffn_train(const uint16_t* xg, const uint16_t* W1, const uint16_t* W3,
                                  const uint16_t* W2, const int32_t* offsets,
                                  const int32_t* counts, uint16_t* h, uint16_t* ab, float* y,
                                  int32_t* dev_status, const moe_shape_t* shape, void* stream);

/* moe_layer_forward over the whole batch (one slice) that leaves in ws (of
 * moe_train_workspace_bytes) everything moe_layer_backward reads: ids, gates,
 * Phi, offsets, counts, route_row, the gathered tokens, h and the
 * pre-activations. out as moe_layer_forward (bitwise the same values).
 * stage_events: NULL or 7 events as in moe_layer_forward. */
moe_status_t moe_layer_forward_train(const float* logits, const uint16_t* x, const uint16_t* W1,
                                     const uint16_t* W3, const uint16_t* W2, uint16_t* out,
                                     void* ws, size_t ws_bytes, int32_t* dev_status,
                                     const moe_shape_t* shape, void* stream,
                                     void* const* stage_events);

/* Pull-reverse-combine: the expert rows pull their upstream gradient through
 * the forward's Phi. dys[row] = dout[src_rank*N + src_idx] (bf16 [moe_rows_max, H],
 * padding rows 0) and gate_row[row] = gates[t, j] for the slot with
 * route_row[t, j] == row (fp32 [moe_rows_max], padding rows 0). A Phi entry
 * that route_row does not point back to raises MOE_DEV_BAD_SCHEDULE. */
moe_status_t moe_reverse_combine(const uint16_t* dout, const int32_t* phi, const int32_t* offsets,
                                 const int32_t* route_row, const float* gates, uint16_t* dys,
                                 float* gate_row, int32_t* dev_status, const moe_shape_t* shape,
                                 void* stream);

/* Activation gradients of the expert FFN (two grouped GEMMs):
 *   dhu = dys . W2[e]^T with the SwiGLU backward fused in its epilogue:
 *     dab: bf16 [moe_rows_max, 2I] = [da | db], hg: bf16 [moe_rows_max, I],
 *     dgate_part: fp32 [moe_rows_max, I/128], the gate gradient of each row
 *     as I/128 partial sums over consecutive 128-column blocks (summed in
 *     order by moe_router_backward);
 *   dxg = [da | db] . [W1[e] | W3[e]]^T: fp32 [moe_rows_max, H].
 * ab and h as left by moe_expert_ffn_train; offsets/counts as for the FFN. */
moe_status_t moe_expert_ffn_dgrad(const uint16_t* dys, const float* gate_row, const uint16_t* ab,
                                  const uint16_t* h, const uint16_t* W1, const uint16_t* W3,
                                  const uint16_t* W2, const int32_t* offsets,
                                  const int32_t* counts, uint16_t* dab, uint16_t* hg,
                                  float* dgate_part, float* dxg, int32_t* dev_status,
                                  const moe_shape_t* shape, void* stream);

/* Push-reverse-dispatch: dx[t] = bf16_rne(acc), acc = 0.0f, acc += dxg[route_row[t,j]]
 * for j = 0..k-1 in ascending order. dx: bf16 [P*N, H]. */
moe_status_t moe_reverse_dispatch(const float* dxg, const int32_t* route_row, uint16_t* dx,
                                  int32_t* dev_status, const moe_shape_t* shape, void* stream);

/* Router gradient: dgate[t,j] = sum of dgate_part[route_row[t,j], 0..I/128-1] in
 * ascending order; S = sum_j gates[t,j] dgate[t,j] (fmaf, ascending j);
 * dlogits[t, ids[t,j]] = gates[t,j] * (dgate[t,j] - S); all other entries 0.
 * dlogits: fp32 [P*N, E]. */
moe_status_t moe_router_backward(const float* dgate_part, const int32_t* route_row,
                                 const int32_t* ids, const float* gates, float* dlogits,
                                 int32_t* dev_status, const moe_shape_t* shape, void* stream);

/* Weight gradients, accumulated per expert over the rows it received in one
 * pass (K = the expert's real rows, rounded up to 64 with zero padding rows):
 *   dW2[e] = hg^T . dys  (fp32 [E, I, H]),
 *   dW1[e] = xg^T . da, dW3[e] = xg^T . db  (fp32 [E, H, I]).
 * Every entry of the three arrays is written. */
moe_status_t moe_expert_ffn_wgrad(const uint16_t* xg, const uint16_t* dys, const uint16_t* dab,
                                  const uint16_t* hg, const int32_t* offsets,
                                  const int32_t* counts, float* dW1, float* dW3, float* dW2,
                                  int32_t* dev_status, const moe_shape_t* shape, void* stream);

/* The whole backward on the state moe_layer_forward_train left in ws (same
 * shape, nothing else written to ws in between): reverse combine, the two
 * activation-gradient GEMMs, reverse dispatch, router gradient, then the
 * weight-gradient GEMMs, all on `stream`. dout: bf16 [P*N, H] upstream
 * gradient; outputs dx bf16 [P*N, H], dlogits fp32 [P*N, E], dW1/dW3 fp32
 * [E, H, I], dW2 fp32 [E, I, H]. stage_events: NULL or 8 events recorded at
 * the start and after each of: reverse combine, dh GEMM, dx GEMM, reverse
 * dispatch, router gradient, dW2 GEMM, dW1|dW3 GEMM. */
moe_status_t moe_layer_backward(const uint16_t* dout, const uint16_t* W1, const uint16_t* W3,
                                const uint16_t* W2, uint16_t* dx, float* dlogits, float* dW1,
                                float* dW3, float* dW2, void* ws, size_t ws_bytes,
                                int32_t* dev_status, const moe_shape_t* shape, void* stream,
                                void* const* stage_events);

/* ------------------------------------------------------------------------
 * MXFP8 ("Mixture-of-Kittens", section 5: MXFP8 routed experts, with the
 * quantisation fused into the dispatch; the OCP Microscaling formats, MXFP8
 * with E4M3 elements): quantisation of rows and of expert weights, the
 * quantising dispatch, the block-scaled expert FFN and the MXFP8 layer.
 *
 * For every block of 32 consecutive values of a row: amax = max |v|, the
 * shared exponent e = floor(log2 amax) - 8 clamped to [-127, 127] (-127 for
 * an all-zero block), the scale stored as the E8M0 code e + 127 and each
 * element as the E4M3 code of v * 2^-e (nearest, ties to even, magnitudes
 * above 448 clamped to 448). The codes depend only on the inputs.
 * ------------------------------------------------------------------------ */

/* Rows of bf16 to MXFP8: src [n_rows, K] (K a multiple of 32) -> q uint8
 * [n_rows, K] E4M3 codes and scale uint8 [n_rows, K/32] E8M0 codes. */
moe_status_t moe_mx_quantize_rows(const uint16_t* src, int64_t n_rows, int32_t K, uint8_t* q,
                                  uint8_t* scale, void* stream);

/* The pull dispatch of moe_dispatch with the MXFP8 quantisation fused: row
 * `row` of xq (uint8 [moe_rows_max, H]) and xs (uint8 [moe_rows_max, H/32])
 * is the quantised token x[src_rank*N + src_idx], (src_rank, src_idx) =
 * phi[row]; padding rows are zero codes with scale code 0. H % 32 == 0.
 * Errors as moe_dispatch. */
moe_status_t moe_dispatch_mxfp8(const uint16_t* x, const int32_t* phi, const int32_t* offsets,
                                uint8_t* xq, uint8_t* xs, int32_t* dev_status,
                                const moe_shape_t* shape, void* stream);

/* The TILED scale layout the block-scaled tensor cores read. For a code
 * matrix [R, K] (R and K multiples of 128; block b covers values 32b..32b+31
 * of a row) the scale of row r, block b is the byte at
 *   ((r / 128) * (K / 128) + b / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + b % 4,
 * i.e. 512-byte atoms of 128 rows x 4 blocks, the K-atoms of a 128-row block
 * consecutive. The table has R * K / 32 bytes, as the row-major one. */

/* moe_dispatch_mxfp8 with xs in the TILED layout of the [moe_rows_max, H]
 * code matrix. H % 128 == 0 (rows_max is a multiple of 256), else
 * MOE_UNSUPPORTED_SHAPE; other errors as moe_dispatch. */
moe_status_t moe_dispatch_mxfp8_tiled(const uint16_t* x, const int32_t* phi,
                                      const int32_t* offsets, uint8_t* xq, uint8_t* xs,
                                      int32_t* dev_status, const moe_shape_t* shape,
                                      void* stream);

/* Expert weights to the MXFP8 operands of the block-scaled FFN: W bf16
 * [E, K, N] (N contiguous) -> q uint8 [E, N, K], the E4M3 codes TRANSPOSED
 * (K contiguous), and scale uint8 [E*N*K/32], the E8M0 codes of the blocks
 * of 32 along K (W[e, 32b..32b+31, n]) in the TILED layout of the [E*N, K]
 * code matrix (row e*N + n). For W1 and W3 (K = H, N = I) and W2 (K = I,
 * N = H); done once per set of weights. Errors: MOE_INVALID_ARG if K or N is
 * not a positive multiple of 128, E < 0, or a pointer is null (E > 0) or not
 * 16-byte aligned (W, q); MOE_UNSUPPORTED_SHAPE if E*K*N >= 2^40. */
moe_status_t moe_mx_quantize_weights(const uint16_t* W, int32_t E, int32_t K, int32_t N,
                                     uint8_t* q, uint8_t* scale, void* stream);

/* Step 3b on MXFP8 operands ("Mixture-of-Kittens", section 5), two kernels
 * on the block-scaled tensor cores (tcgen05.mma kind::mxf8f6f4.block_scale,
 * fp32 accumulation in a fixed K order):
 *   GEMM1: for row r of expert l's segment, a = mx(xq[r]) . mx(W1[l]),
 *          b = mx(xq[r]) . mx(W3[l]) (fp32), h = silu(a) * b (fp32), written
 *          as MXFP8 along I: hq uint8 [moe_rows_max, I] codes and hs the
 *          TILED scales of that matrix (the dispatch's quantisation rule
 *          applied to the fp32 h);
 *   GEMM2: y[r] = mx(hq[r]) . mx(W2[l]), fp32 [moe_rows_max, H];
 * mx(.) = code value x 2^(scale code - 127). xq/xs: moe_dispatch_mxfp8_tiled's
 * outputs; W1q/W1s, W3q/W3s, W2q/W2s: moe_mx_quantize_weights of W1, W3, W2.
 * Requires the moe_expert_ffn limits and pad % 256 == 0 (CTA-pair tiles).
 * hq, y 32-byte aligned, every other pointer 16-byte aligned. Rows of tiles
 * holding only padding are not written, nor y of 32-row blocks past the last
 * route of their expert. Errors as moe_expert_ffn. */
moe_status_t moe_expert_ffn_mxfp8(const uint8_t* xq, const uint8_t* xs, const uint8_t* W1q,
                                  const uint8_t* W1s, const uint8_t* W3q, const uint8_t* W3s,
                                  const uint8_t* W2q, const uint8_t* W2s, const int32_t* offsets,
                                  const int32_t* counts, uint8_t* hq, uint8_t* hs, float* y,
                                  int32_t* dev_status, const moe_shape_t* shape, void* stream);

/* Workspace of moe_layer_forward_mxfp8 with a shared expert: the layer's
 * workspace plus the shared expert's h (bf16) and output (fp32) over every
 * token (and a padded copy of x when P*N % 256 != 0). 0 if the shape is not
 * supported. */
size_t moe_layer_mxfp8_workspace_bytes(const moe_shape_t* shape);

/* Steps 1-4 with MXFP8 routed experts: route, schedule, the quantising
 * dispatch (TILED scales), moe_expert_ffn_mxfp8 and the fixed-order combine,
 * on `stream`; the dispatch runs inside GEMM1 (a spare warp of every CTA
 * quantises 128-row blocks of x[Phi[row]] while the tensor cores consume
 * earlier ones), with the results of moe_dispatch_mxfp8_tiled.
 * Routed weights as moe_expert_ffn_mxfp8.
 * Ws1, Ws3 bf16 [H, I] and Ws2 bf16 [I, H] (all three, or all null): a bf16
 * shared expert ("Mixture-of-Kittens", section 5) every token passes through,
 * ys[t] = bf16(silu(x[t].Ws1) * (x[t].Ws3)).Ws2 in fp32 on the bf16 FFN's
 * kernels; the combine then starts each token's fixed-order sum from it:
 *   acc = ys[t]; acc = fmaf(g[t,j], y[route_row[t,j]], acc), j = 0..k-1;
 *   out[t] = bf16_rne(acc).
 * ws: moe_layer_workspace_bytes without a shared expert (the codes and scales
 * of x and h take the places of xg and h), moe_layer_mxfp8_workspace_bytes
 * with one. stage_events as moe_layer_forward (the shared expert falls
 * between the third and fourth). Limits as moe_expert_ffn_mxfp8. */
moe_status_t moe_layer_forward_mxfp8(const float* logits, const uint16_t* x, const uint8_t* W1q,
                                     const uint8_t* W1s, const uint8_t* W3q, const uint8_t* W3s,
                                     const uint8_t* W2q, const uint8_t* W2s, const uint16_t* Ws1,
                                     const uint16_t* Ws3, const uint16_t* Ws2, uint16_t* out,
                                     void* ws, size_t ws_bytes, int32_t* dev_status,
                                     const moe_shape_t* shape, void* stream,
                                     void* const* stage_events);

/* Number of kernels this library has launched in the calling process. */
int64_t moe_launch_count(void);

/* Failure-detection self test: launches one kernel that waits, with the same
 * bounded wait the FFN pipeline uses, on an mbarrier that nothing completes,
 * giving up after timeout_ns nanoseconds; it then raises MOE_DEV_TIMEOUT in
 * *dev_status. The context stays usable. */
moe_status_t moe_selftest_bounded_wait(int32_t* dev_status, int64_t timeout_ns, void* stream);

/* Failure-detection self test of the schedule's one-launch kernel
 * (moe_schedule runs it when all its blocks fit on the device at once; its
 * grid barrier is a bounded wait): the same kernel, on the same
 * arguments as moe_schedule, with a barrier that waits for one block more
 * than the launch has. Every block gives up after timeout_ns nanoseconds,
 * raises MOE_DEV_TIMEOUT in *dev_status and returns; the outputs are then
 * incomplete and the context stays usable. MOE_UNSUPPORTED_SHAPE if the
 * shape does not take the one-launch kernel; N >= 1. */
moe_status_t moe_selftest_schedule_barrier(const int32_t* ids, int32_t* phi, int32_t* offsets,
                                           int32_t* counts, int32_t* route_row, void* ws,
                                           size_t ws_bytes, int32_t* dev_status,
                                           const moe_shape_t* shape, int64_t timeout_ns,
                                           void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
