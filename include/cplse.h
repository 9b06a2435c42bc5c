/*
 * cplse: the data-parallel hot path of decode-context-parallel (DCP) attention
 * and of Ulysses sequence parallelism, for NVIDIA B200 (sm_100a).
 *
 *   pack     form LSE = softmax_max + log(softmax_sum) while writing the
 *            head-partitioned send packet (payload in one region, fp32 LSE in
 *            another); invalid statistics give LSE = -inf
 *   a2a      the all-to-all's block permutation, W ranks emulated on one GPU
 *   combine  stable log-sum-exp merge of the W partial outputs
 *   fused    pack -> a2a -> combine in one pass; the packet never exists
 *   Ulysses  sequence-scatter/head-gather layout transform and its inverse
 *
 * Sources, cited by page title and section:
 *  [DCP] vLLM-Ascend pull request "[Performance][Attention] Fuse local SFA LSE
 *        formation into DCP pack", sections "What this PR does / why we need
 *        it?" (Before/After pipelines: native fp32 softmax_max/softmax_sum ->
 *        max/sum-aware DCP pack -> HCCL All2All -> stable combine; invalid
 *        statistics) and "How was this patch tested?" (bf16 and fp16,
 *        scatter_dim 0 and 1, head dim 512, non-contiguous output/max/sum
 *        strides, graph capture with changed-input replay).
 *  [ULY] FastVideo compare view "[perf] Probe H3 chunked all-to-all with
 *        direct output slices": all_to_all_4D(x, 2, 1) maps [B, S/W, H, D] to
 *        [B, S, H/W, D] and all_to_all_4D(x, 1, 2) maps back; results must be
 *        byte-identical to the NCCL all-to-all.
 *
 * Conventions for every entry point:
 *  - Notation: W ranks, T tokens, H heads, Hc = H / W, D head dim. Layouts
 *    are row-major, last index fastest. A "row" is the D elements of one
 *    (rank, token, head). Payload elements are bf16 or fp16 (2 bytes).
 *  - Pointers are DEVICE pointers on the current CUDA device (host pointers
 *    are rejected with CP_ERR_ARG). The caller allocates and owns every
 *    buffer; the library never allocates, frees or synchronises.
 *  - `stream` is a cudaStream_t (NULL: the legacy default stream). Calls only
 *    enqueue work on it and return; results are ready when the stream is.
 *    No call performs a host<->device copy or a host synchronisation.
 *  - Outputs must not overlap inputs (CP_ERR_ALIAS).
 *  - All validation happens on the host before any launch. A failing call
 *    enqueues nothing, returns a negative cp_status and records a message
 *    for cp_last_error(). A call with zero rows (T == 0 or B == 0) is a
 *    valid no-op. The library never aborts the process and has no device
 *    side traps, asserts or waits.
 */
#ifndef CPLSE_H
#define CPLSE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define CPLSE_API __attribute__((visibility("default")))
#else
#define CPLSE_API
#endif

#define CPLSE_ABI_VERSION 4
#define CPLSE_MAX_W 32     /* simulated ranks per call */
#define CPLSE_MAX_D 1024   /* head dim, elements */

typedef enum cp_status {
    CP_OK = 0,
    CP_ERR_ARG = -1,          /* null/host pointer, bad enum, negative size */
    CP_ERR_SHAPE = -2,        /* H % W, T % W, S_local, D % 8 ... */
    CP_ERR_ALIGN = -3,        /* base not 16-byte aligned, stride not a multiple of 8 elements */
    CP_ERR_ALIAS = -4,        /* an output overlaps an input */
    CP_ERR_UNSUPPORTED = -5,  /* W > 32, D > 1024, ... */
    CP_ERR_CUDA = -6          /* the launch itself failed (message has the CUDA error) */
} cp_status;

typedef enum cp_dtype { CP_BF16 = 0, CP_FP16 = 1 } cp_dtype;

/* Element strides of a [W][T][H] (or [W][T][H][D] with D contiguous) view. */
typedef struct cp_strides3 {
    int64_t r, t, h;
} cp_strides3;

/* CPLSE_ABI_VERSION of the loaded library. */
CPLSE_API int cp_abi_version(void);

/* Message of the last failing call on this host thread ("" if none). The
 * pointer stays valid until the next call on the same thread. */
CPLSE_API const char* cp_last_error(void);

/*
 * [DCP] After pipeline: the pack itself turns each row's (max, sum) into its
 * LSE, in the same pass that moves the row's payload into the packet, so no
 * separate LSE tensor exists. Statistics that cannot describe a softmax (max
 * not finite, sum not finite, or sum not positive) give LSE = -inf; otherwise
 * LSE = max + logf(sum), in fp32.
 *
 *   o      payload [W][T][H][D], element strides `so` (D contiguous; so.* >= 0
 *          and multiples of 8; base 16-byte aligned)
 *   smax   fp32 [W][T][H], element strides `sm` (>= 0, any value)
 *   ssum   fp32 [W][T][H], element strides `ss`
 *   scatter_dim 1 (head chunks, the DCP path; H % W == 0):
 *            pkt_o   [W_src][W_dst][T][Hc][D]   pkt_o[r][j][t][hc] = o[r][t][j*Hc+hc]
 *            pkt_lse [W_src][W_dst][T][Hc]      fp32
 *   scatter_dim 0 (token chunks; T % W == 0, Tc = T / W):
 *            pkt_o   [W_src][W_dst][Tc][H][D]   pkt_o[r][j][tc][h] = o[r][j*Tc+tc][h]
 *            pkt_lse [W_src][W_dst][Tc][H]
 *   Payload bits are copied unchanged. pkt_o: 16-byte aligned, contiguous.
 */
CPLSE_API cp_status cp_pack_lse(const void* o, cp_strides3 so, const float* smax, cp_strides3 sm,
                      const float* ssum, cp_strides3 ss, int W, int64_t T, int H, int D,
                      cp_dtype dt, int scatter_dim, void* pkt_o, float* pkt_lse, void* stream);

/*
 * [DCP] Before pipeline, first step: LSE computed from max and sum into a
 * tensor of its own. The pull request keeps this older path alongside the new
 * pack; here it is the A/B baseline of the max/sum-aware pack.
 * Writes a standalone fp32 tensor lse [W][T][H] (contiguous) with the same
 * values cp_pack_lse forms (max + logf(sum), -inf for invalid statistics).
 *   smax, ssum fp32 [W][T][H], element strides sm / ss (>= 0).
 */
CPLSE_API cp_status cp_lse_materialize(const float* smax, cp_strides3 sm, const float* ssum,
                                       cp_strides3 ss, int W, int64_t T, int H, float* lse,
                                       void* stream);

/*
 * [DCP] Before pipeline, remaining steps (rearranging into packet order, then
 * packing): the same packet as cp_pack_lse, but its LSE region is a copy of a
 * materialized LSE tensor (element strides sl) moved into the packet layout,
 * instead of being formed from max/sum. cp_lse_materialize followed by this
 * call gives the packet of cp_pack_lse bit for bit.
 */
CPLSE_API cp_status cp_pack_from_lse(const void* o, cp_strides3 so, const float* lse,
                                     cp_strides3 sl, int W, int64_t T, int H, int D, cp_dtype dt,
                                     int scatter_dim, void* pkt_o, float* pkt_lse, void* stream);

/*
 * [DCP] The all-to-all of the packet (HCCL on the page's hardware), emulated
 * on one GPU: W simulated ranks
 * each hold W blocks of `block_bytes`; block j of rank r lands as block r of
 * rank j:  recv[j][r] = send[r][j]. Call it once per packet region (payload
 * block = T*Hc*D*2 bytes, LSE block = T*Hc*4 bytes). Any block size works;
 * 16-byte aligned bases with block_bytes % 16 == 0 take the vector path.
 */
CPLSE_API cp_status cp_a2a_local_permute(const void* send, void* recv, int W, int64_t block_bytes,
                               void* stream);

/*
 * [DCP] the stable combine each destination rank runs on what it received.
 *   recv_o   [W_dst][W_src][N][D] payload, N = T*Hc rows per block
 *   recv_lse [W_dst][W_src][N]    fp32, each finite or -inf (NaN counts as -inf)
 *   out      [W_dst][N][D]        payload dtype, fp32 accumulation, nearest-even
 *   out_lse  [W_dst][N]           fp32
 * Per output row, over r = 0..W-1: M = max lse_r; if M = -inf the row is all
 * invalid: out = +0, out_lse = -inf. Otherwise LSE* = M + logf(sum_r expf(lse_r - M)),
 * out = sum_r expf(lse_r - LSE*) * o_r over the valid r only (an invalid
 * contribution's payload is never read into the sum). For the token-chunk
 * packet pass T/W as T and H as Hc.
 */
CPLSE_API cp_status cp_lse_combine(const void* recv_o, const float* recv_lse, int W, int64_t T, int Hc,
                         int D, cp_dtype dt, void* out, float* out_lse, void* stream);

/*
 * pack -> a2a -> combine in one pass: each output row reads its source row of
 * every rank's o/smax/ssum directly, so the packet never exists. Inputs as in
 * cp_pack_lse. Outputs are what cp_lse_combine gives on the received packet:
 *   scatter_dim 1 (head chunks; H % W == 0): destination j holds heads
 *            j*Hc .. j*Hc+Hc-1 of every token:
 *            out [W][T][Hc][D], out_lse [W][T][Hc]; row (j, t, hc) reads (t, j*Hc + hc)
 *   scatter_dim 0 (token chunks; T % W == 0, Tc = T / W): destination j holds
 *            tokens j*Tc .. j*Tc+Tc-1 with all heads:
 *            out [W][Tc][H][D], out_lse [W][Tc][H]; row (j, tc, h) reads (j*Tc + tc, h),
 *            i.e. [T][H] in source order
 * Bit-identical to cp_pack_lse(scatter_dim) -> cp_a2a_local_permute (both
 * regions) -> cp_lse_combine (with T/W as T and H as Hc for token chunks).
 * out: 16-byte aligned, contiguous; out_lse: 4-byte aligned, contiguous.
 */
CPLSE_API cp_status cp_pack_permute_combine_fused(const void* o, cp_strides3 so, const float* smax,
                                        cp_strides3 sm, const float* ssum, cp_strides3 ss, int W,
                                        int64_t T, int H, int D, cp_dtype dt, int scatter_dim,
                                        void* out, float* out_lse, void* stream);

/*
 * ---- One process per GPU: the exchange across W real ranks ----------------
 *
 * [DCP] The pipeline's all-to-all is a real collective when every rank is its
 * own GPU: rank r holds the partial output of KV shard r (o [T][H][D] and its
 * max/sum [T][H]); destination j receives head chunk j (or token chunk j) of
 * every rank and combines it. Two ways to run it on B200:
 *   a2a:  cp_pack_lse_rank -> an all-to-all of both packet regions (NCCL,
 *         equal W-way splits) -> cp_lse_combine_rank;
 *   pull: cp_pull_combine, one kernel per destination that loads the rows it
 *         merges from every rank's o/max/sum where they live (peer memory
 *         mapped into this process), so that no packet exists anywhere.
 * All three give, on rank j, destination j's block of
 * cp_pack_permute_combine_fused's output for the same W planes, bit for bit.
 */

/*
 * Mapping another rank's buffers into this process for cp_pull_combine (CUDA
 * IPC of plain device memory; no multicast, no fabric handles). The owner
 * exports the address of a buffer it allocated with cudaMalloc (a caching
 * allocator's block is fine: the handle names the whole allocation and the
 * offset locates the buffer in it); the handle is plain bytes that the caller
 * moves to the other processes of the same node. A reader imports it with its
 * own device current: the owner's memory becomes addressable by the reader's
 * kernels (peer access is enabled as needed). `base` is what cp_ipc_close
 * takes once the reader is done; the owner must keep the buffer allocated
 * until every reader has closed it. A handle cannot be imported by the
 * process that exported it (CP_ERR_CUDA).
 */
typedef struct cp_ipc_handle {
    unsigned char handle[64];   /* cudaIpcMemHandle_t of the allocation */
    int64_t offset;             /* bytes from the allocation's start to the buffer */
    int64_t alloc_bytes;        /* size of the allocation */
    int32_t device;             /* the owner's device ordinal */
    int32_t reserved;
} cp_ipc_handle;

CPLSE_API cp_status cp_ipc_export(const void* p, cp_ipc_handle* h);
CPLSE_API cp_status cp_ipc_import(const cp_ipc_handle* h, void** base, void** p);
CPLSE_API cp_status cp_ipc_close(void* base);

/*
 * [DCP] After pipeline, one real rank: the pack of cp_pack_lse for a single
 * source plane. o [T][H][D] (strides so.t, so.h; so.r ignored), smax / ssum
 * [T][H] fp32 (strides .t, .h; .r ignored). W is the number of destination
 * ranks. Writes this rank's send packet, destination-major:
 *   scatter_dim 1: pkt_o [W_dst][T][Hc][D], pkt_lse [W_dst][T][Hc]
 *   scatter_dim 0: pkt_o [W_dst][T/W][H][D], pkt_lse [W_dst][T/W][H]
 * equal to plane r of cp_pack_lse's packet for the same W planes. Each
 * region splits into W equal contiguous blocks, one per destination, as an
 * all-to-all with equal splits expects.
 */
CPLSE_API cp_status cp_pack_lse_rank(const void* o, cp_strides3 so, const float* smax,
                                     cp_strides3 sm, const float* ssum, cp_strides3 ss, int W,
                                     int64_t T, int H, int D, cp_dtype dt, int scatter_dim,
                                     void* pkt_o, float* pkt_lse, void* stream);

/*
 * [DCP] The stable combine on one real destination rank, after the
 * all-to-all: recv_o [W_src][N][D], recv_lse [W_src][N] (N = T*Hc rows; for
 * token chunks pass T/W as T and H as Hc) -> out [N][D], out_lse [N]. Same
 * rule and same bits as cp_lse_combine for one destination.
 */
CPLSE_API cp_status cp_lse_combine_rank(const void* recv_o, const float* recv_lse, int W,
                                        int64_t T, int Hc, int D, cp_dtype dt, void* out,
                                        float* out_lse, void* stream);

/*
 * [DCP] pack -> all-to-all -> combine for destination `dst` of W real ranks,
 * in one kernel on dst's GPU, pulling each source row over NVLink.
 *   o, smax, ssum  HOST arrays of W device addresses: rank r's o [T][H][D]
 *                  and max/sum [T][H] planes. Each address must be usable by
 *                  the current device: its own memory, or a peer's mapped into
 *                  this process (CUDA IPC) with peer access between the two.
 *                  Every plane has the layout given by so / sm / ss (.t, .h;
 *                  .r ignored).
 *   scatter_dim 1: out [T][Hc][D], out_lse [T][Hc]: heads dst*Hc .. of every token
 *   scatter_dim 0: out [T/W][H][D], out_lse [T/W][H]: tokens dst*T/W .. with all heads
 * The kernel reads the planes with ordinary 16-byte loads (no bulk or
 * multicast copies) and waits for nothing: the caller orders it after every
 * rank's writes to its planes and before any rank overwrites them again (a
 * stream-ordered barrier such as a one-element all-reduce on both sides).
 */
CPLSE_API cp_status cp_pull_combine(const void* const* o, cp_strides3 so,
                                    const float* const* smax, cp_strides3 sm,
                                    const float* const* ssum, cp_strides3 ss, int W, int64_t T,
                                    int H, int D, cp_dtype dt, int scatter_dim, int dst,
                                    void* out, float* out_lse, void* stream);

/*
 * [ULY] all_to_all_4D(x, scatter_dim=2, gather_dim=1), W ranks on one GPU:
 *   in  [W][B][S_local][H][D]  ->  out [W][B][W*S_local][H/W][D]
 *   out[j][b][r*S_local + s][hc] = in[r][b][s][j*Hc + hc]
 * A byte copy of elem_bytes-sized elements (1, 2, 4 or 8); H % W == 0.
 */
CPLSE_API cp_status ulysses_seq2head(const void* in, void* out, int W, int B, int64_t S_local, int H, int D,
                           int elem_bytes, void* stream);

/*
 * [ULY] all_to_all_4D(x, scatter_dim=1, gather_dim=2), the inverse:
 *   in  [W][B][W*S_local][H/W][D]  ->  out [W][B][S_local][H][D]
 *   out[j][b][s][r*Hc + hc] = in[r][b][j*S_local + s][hc]
 * ulysses_head2seq(ulysses_seq2head(x)) == x.
 */
CPLSE_API cp_status ulysses_head2seq(const void* in, void* out, int W, int B, int64_t S_local, int H, int D,
                           int elem_bytes, void* stream);

/*
 * [ULY] The Ulysses all-to-alls across W real ranks, one per GPU, as a
 * load/store exchange over NVLink: destination `dst` reads its share of every
 * rank's tensor where it lives and writes its own result, byte-identical to
 * the NCCL all_to_all_4D and to block dst of the single-GPU calls above.
 *   in   HOST array of W device addresses: rank r's tensor (this device's
 *        memory, or a peer's mapped into this process with cp_ipc_import)
 *   out  destination dst's tensor, on the current device
 * seq2head: in[r] [B][S_local][H][D] -> out [B][W*S_local][H/W][D],
 *           out[b][r*S_local + s][hc] = in[r][b][s][dst*Hc + hc]
 * head2seq: in[r] [B][W*S_local][H/W][D] -> out [B][S_local][H][D],
 *           out[b][s][r*Hc + hc] = in[r][b][dst*S_local + s][hc]
 * Ordinary loads and stores only (no bulk or multicast copies); the caller
 * orders the call after every rank's writes to its tensor and before any
 * rank overwrites it again. B <= 65535.
 */
CPLSE_API cp_status ulysses_seq2head_pull(const void* const* in, void* out, int W, int B,
                                          int64_t S_local, int H, int D, int elem_bytes, int dst,
                                          void* stream);
CPLSE_API cp_status ulysses_head2seq_pull(const void* const* in, void* out, int W, int B,
                                          int64_t S_local, int H, int D, int elem_bytes, int dst,
                                          void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CPLSE_H */
