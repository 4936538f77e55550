/*
 * lvsa.h -- C ABI of the B200 (sm_100a) library for LVSA frame-granular
 * block-sparse self-attention.
 *
 * Method: "LVSA: Training-Free Sparse Attention for Long Video Diffusion".
 * A query frame t of a video of T latent frames attends only to the frames of
 *     A(t) = G_s U W(t)
 * (gist.science technical summary, section 2 "Core Mechanism"): G_s are
 * G = C - W global anchor frames whose offset rotates with the denoising step
 * s, W(t) is a local window of W frames that is extended until |A(t)| reaches
 * the budget C (same summary, "Rotating Global Anchors" and "Expanded Adaptive
 * Windows"; techwalker article "华为巴黎研究院让AI视频“不再原地打转”", sections
 * 二 and 三).
 *
 * Conventions for every entry point:
 *  - Every function returns an lvsa_status; nothing is thrown, nothing aborts.
 *  - Arguments are validated before any CUDA call or launch; on an error return
 *    no output has been written and nothing was launched.
 *  - The library never allocates device memory at run time and never frees
 *    caller memory: the caller owns every buffer it passes (lvsa_ipc_import
 *    maps another process's buffer; lvsa_ipc_release unmaps it).  The one
 *    static device array of lvsa_attention_host_static is part of the loaded
 *    module.
 *  - Thread safety: lvsa_build_frame_lists is pure; lvsa_attention and
 *    lvsa_attention_host may be called from several host threads.
 */
#ifndef LVSA_H
#define LVSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LVSA_OK = 0,
  LVSA_ERR_INVALID_ARG = 1,      /* a size, pointer or parameter is out of range */
  LVSA_ERR_UNSUPPORTED = 2,      /* valid but not supported here (e.g. head dim not 64/128, no sm_100 device) */
  LVSA_ERR_CUDA = 3,             /* a CUDA runtime/driver call failed */
  LVSA_ERR_TIMEOUT = 4,          /* a device-side bounded wait ran out (see lvsa_get_device_status) */
  LVSA_ERR_BUFFER_TOO_SMALL = 5, /* the output capacity is below what the call must write */
  LVSA_ERR_BAD_LIST = 6          /* a device frame list held an entry outside [0, T) */
} lvsa_status;

/* Device status bits reported by lvsa_get_device_status. */
#define LVSA_DEV_TIMEOUT  0x1u   /* a kernel's bounded wait expired; that CTA stopped early */
#define LVSA_DEV_BAD_LIST 0x2u   /* a frame-list entry was outside [0, T); the entry was skipped */

/*
 * lvsa_build_frame_lists -- per-query-frame KV frame lists A(t) for step `step`.
 *
 * Defines: A(t) = G_s U W(t) (gist.science summary, section 2 "Core
 * Mechanism"), with
 *   - G = C - W anchors at spacing about T / (C - W) (techwalker article,
 *     section 二), placed at floor(k*T/G), k = 0..G-1, shifted by step mod T
 *     (same article, section 三: one frame per step, modulo the total frame
 *     count);
 *   - the window of W frames centred on t (lo = t - W/2), shifted inward at the
 *     sequence ends;
 *   - extension (gist.science summary, "Expanded Adaptive Windows"; techwalker
 *     article, section 二): new non-anchor frames are added alternately right
 *     then left of the window until |A(t)| = C; a side at the sequence end is
 *     skipped;
 *   - C >= T: every row is 0..T-1 (dense attention).
 *
 * Arguments:
 *   T, C, W  latent frames, frame budget, window size; need T >= 1, 1 <= W <= C.
 *   step     denoising step, >= 0.
 *   out      HOST int32 buffer, caller-owned, row-major [T][L] with
 *            L = min(C, T); each row strictly ascending frame indices in [0,T).
 *   out_capacity  number of int32 elements `out` can hold (>= T*L).
 *   out_L    optional (may be NULL): receives L.
 * Errors: LVSA_ERR_INVALID_ARG (parameters), LVSA_ERR_BUFFER_TOO_SMALL (capacity;
 *   *out_L is still set so the caller can size the buffer; out may be NULL then).
 * Host only; no CUDA call; cost O(T*C).
 */
lvsa_status lvsa_build_frame_lists(int T, int C, int W, long long step,
                                   int32_t* out, size_t out_capacity, int* out_L);

/*
 * lvsa_build_anchors -- the G = C - W anchor frames of step `step`, ascending
 * (techwalker article, section 三; gist.science summary, "Rotating Global
 * Anchors").  out: HOST int32 buffer of out_capacity elements (>= G).
 * *out_G receives G (0 when C >= T or W == C: no anchors).
 * Errors as lvsa_build_frame_lists.
 */
lvsa_status lvsa_build_anchors(int T, int C, int W, long long step,
                               int32_t* out, size_t out_capacity, int* out_G);

/*
 * lvsa_attention -- frame-granular block-sparse softmax attention.
 *
 * Defines (gist.science summary, section 2 "Core Mechanism" and "Complexity";
 * page 1 "LVSA hoạt động như thế nào": block-sparse attention over structured
 * windows plus rotating anchors): for query token i of frame t, batch b, head h
 *     out[b,i,h,:] = sum_j softmax_j(scale * q[b,i,h,:] . k[b,j,h,:]) v[b,j,h,:]
 * with j running over the tokens of the frames listed in lists[t][0..L-1],
 * one softmax over all of them together.  Cost O(T * L * P^2 * d) per head.
 *
 * Arguments:
 *   q, k, v  DEVICE bf16, contiguous [batch][T*tokens_per_frame][heads][d]
 *            (frame-major tokens: token t*P + i is patch i of frame t), 16-byte
 *            aligned.  Values must be finite.
 *   lists    DEVICE int32 [T][L], row t = the frames attended by query frame t
 *            (as written by lvsa_build_frame_lists, or 0..T-1 in every row for
 *            dense attention).  A row is a set: order and repeated entries do
 *            not matter.  Entries outside [0,T) are skipped and flag
 *            LVSA_DEV_BAD_LIST; a frame with no valid entry gets a zero output.
 *   L        list width, 1 <= L <= T.
 *   T, tokens_per_frame (P), heads (H), d, batch: sizes; d must be 64 or 128;
 *            T <= 4096 (LVSA_ERR_UNSUPPORTED above).
 *   scale    softmax scale; <= 0 selects 1/sqrt(d).
 *   out      DEVICE bf16, same layout as q, 16-byte aligned, must not overlap
 *            q, k, v or lists.
 *   stream   a cudaStream_t (passed as void*), NULL = default stream.
 * Behaviour: asynchronous on `stream`; returns after the launch.  Argument and
 * launch errors are returned here.  A device-side wait that runs out (a hung
 * pipeline) stops that CTA, sets LVSA_DEV_TIMEOUT, and is reported by
 * lvsa_get_device_status after the stream is synchronised.
 * Needs an sm_100 (B200-class) device; otherwise LVSA_ERR_UNSUPPORTED.
 * The call can be captured into a CUDA graph (the tensor maps travel by value
 * in the launch parameters; a replay reads whatever the same buffers hold).
 */
lvsa_status lvsa_attention(const void* q, const void* k, const void* v,
                           const int32_t* lists, int L, int T, int tokens_per_frame,
                           int heads, int d, int batch, float scale,
                           void* out, void* stream);

/*
 * lvsa_attention_joint -- lvsa_attention over a joint video + text sequence:
 * [batch][T*tokens_per_frame + text_tokens][heads][d], the text tokens after
 * the frame-major video tokens (the joint attention of a dual-stream model
 * such as HunyuanVideo 1.5, named in the techwalker article, section 四).
 *
 * Defines (the pages give A(t) for video frames only and say nothing of other
 * tokens; the reading taken): a video query of frame t attends the tokens of
 * the frames in A(t) and every text token; a text query attends every token;
 * one softmax per row.  text_tokens = 0 is lvsa_attention exactly (the same
 * bits).
 *
 * Arguments as lvsa_attention, with text_tokens >= 0 and
 * T*tokens_per_frame + text_tokens <= INT_MAX; q, k, v, out hold the joint
 * sequence.  Behaviour and errors as lvsa_attention.
 */
lvsa_status lvsa_attention_joint(const void* q, const void* k, const void* v,
                                 const int32_t* lists, int L, int T, int tokens_per_frame,
                                 int text_tokens, int heads, int d, int batch, float scale,
                                 void* out, void* stream);

/*
 * lvsa_attention_host -- lvsa_attention on HOST inputs and output, with the
 * transfers pipelined against the kernel by bands of heads.
 *
 * Defines the same output as lvsa_attention.  Heads are independent in the
 * method (the frame lists A(t) are indexed by query frame and step only, and
 * shared by every head and batch entry: gist.science summary, section 2
 * "Core Mechanism"), so the call is cut into bands of heads: band g's Q, K, V
 * columns are copied host -> device, its attention kernel runs, and its output
 * columns are copied device -> host; the upload of band g+1 and the readback
 * of band g-1 overlap the kernel of band g.
 *
 * Arguments:
 *   q_host, k_host, v_host  HOST bf16 [batch][T*tokens_per_frame][heads][d].
 *            Page-locked (pinned) memory is needed for the copies to overlap.
 *   lists_host  HOST int32 [T][L] (as written by lvsa_build_frame_lists).
 *   L, T, tokens_per_frame, heads, d, batch, scale  as lvsa_attention.
 *   out_host HOST bf16, same layout as q_host; must not overlap q/k/v_host or
 *            lists_host.
 *   q_dev, k_dev, v_dev, out_dev  DEVICE staging buffers of the full tensor
 *            size (batch*T*tokens_per_frame*heads*d bf16 each), caller-owned,
 *            16-byte aligned; out_dev must not overlap q/k/v_dev or lists_dev.  On return
 *            from the stream they hold the inputs and the output.
 *   lists_dev   DEVICE int32 [T][L] staging buffer, 4-byte aligned.
 *   heads_per_band  heads per band, 1..heads; 0 = one head per band.
 *   stream   a cudaStream_t (as void*), NULL = default stream.  The copies
 *            start after the work already queued on `stream`; work queued on
 *            `stream` after this call runs after out_host is written.  The
 *            library keeps four internal streams (upload, readback, and two
 *            that the band kernels alternate on) and a set of events per device
 *            (created on first use, never freed); calls are serialised by a
 *            lock while they are queued.
 * Behaviour: asynchronous; errors as lvsa_attention (a failure part-way
 * returns LVSA_ERR_CUDA and leaves out_host partly written).  Synchronise
 * `stream` before reading out_host.  The call can be captured into a CUDA
 * graph on `stream` (the internal streams join the capture through events).
 */
lvsa_status lvsa_attention_host(const void* q_host, const void* k_host, const void* v_host,
                                const int32_t* lists_host, int L, int T, int tokens_per_frame,
                                int heads, int d, int batch, float scale, void* out_host,
                                void* q_dev, void* k_dev, void* v_dev, int32_t* lists_dev,
                                void* out_dev, int heads_per_band, void* stream);

/* Bytes of the device staging array lvsa_attention_host_static works in (64 MiB). */
#define LVSA_STATIC_SCRATCH_BYTES (64ull << 20)

/*
 * lvsa_attention_host_static -- lvsa_attention on HOST inputs and output that
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library call,
 * and no caller-provided device buffer.
 *
 * The paper has no counterpart to this call.  It is for callers that cannot
 * get device memory of their own for staging: a plug-in running inside a
 * process whose allocator already owns the GPU's memory (a framework's caching
 * allocator, or a memory-capped service), or code on a path where cudaMalloc /
 * cudaFree must not be called because they can block or synchronise the whole
 * device.
 *
 * The inputs, the lists and the output are staged in one array of
 * LVSA_STATIC_SCRATCH_BYTES in the library's own device memory (a static
 * __device__ array: every GPU that loads the library holds it until the
 * process exits).  Q, K, V, the lists and the output are copied host -> array
 * -> host on `stream` around one attention launch; the result is the one
 * lvsa_attention computes.
 *
 * Arguments: q_host, k_host, v_host, lists_host, L, T, tokens_per_frame, heads,
 *   d, batch, scale, out_host as lvsa_attention_host (host buffers; pinned
 *   memory lets the copies run asynchronously); stream a cudaStream_t (as
 *   void*), NULL = default stream.
 * Limit: 4 * batch*T*tokens_per_frame*heads*d*2 bytes (Q, K, V, output, each
 *   rounded up to 256 bytes) + T*L*4 bytes (lists, rounded up to 256) must fit
 *   in LVSA_STATIC_SCRATCH_BYTES; a larger call is refused with
 *   LVSA_ERR_INVALID_ARG before anything is copied or launched.
 * Behaviour: asynchronous on `stream`; synchronise it before reading out_host.
 *   The first call on a device looks up the array's device address (one
 *   cudaGetSymbolAddress, with that device current).  Every call on a device
 *   shares the one array, which keeps the previous call's contents (each call
 *   overwrites what it reads before reading it): calls whose work overlaps on
 *   the GPU (other streams, other host threads) race on it -- serialise them,
 *   e.g. on one stream.  Errors as lvsa_attention.
 */
lvsa_status lvsa_attention_host_static(const void* q_host, const void* k_host, const void* v_host,
                                       const int32_t* lists_host, int L, int T, int tokens_per_frame,
                                       int heads, int d, int batch, float scale, void* out_host,
                                       void* stream);

/*
 * Sequence-parallel use (DeepSpeed-Ulysses layout, under which the method runs
 * Wan 2.2-A14B on 8 NPUs: techwalker article, section 五).  N ranks, one per
 * GPU of a node; rank r holds tokens [start_r, start_r + n_r) of the
 * frame-major sequence (n_r = chunk_tokens[r], start_r their prefix sum) of
 * Q, K, V and the output, for every head: [batch][n_r][heads][d] bf16.  Rank r
 * computes attention for a band of heads [head0, head0 + band) over all
 * tokens -- heads are independent because A(t) is shared by every head (gist.science
 * summary, section 2 "Core Mechanism").  Per step:
 *   1. barrier (every rank's inputs written);
 *   2. lvsa_seq_to_heads: gather the band from every rank's range, reading
 *      the other GPUs' buffers through peer mappings (lvsa_ipc_import);
 *   3. lvsa_attention_to_chunks: attention over the band, each output row
 *      stored straight into the range buffer of the rank that owns its token;
 *   4. barrier (every rank's output rows stored).
 * No kernel of this library waits on another GPU; the caller's process group
 * orders the ranks.
 */

/*
 * lvsa_seq_to_heads -- gathers heads [head0, head0 + band) of Q, K and V from
 * token-range buffers into whole-sequence band buffers (a pure copy, bit for
 * bit).
 *
 * Arguments:
 *   q_chunks, k_chunks, v_chunks  HOST arrays of nchunks pointers this GPU can
 *            address (its memory, another GPU's with peer access -- enabled
 *            here if it is not yet -- or a peer mapping, or pinned host memory),
 *            chunk c = [batch][chunk_tokens[c]][heads][d] bf16, 16-byte aligned;
 *            may be NULL where chunk_tokens[c] == 0.  A pointer the GPU cannot
 *            address (pageable host memory, another GPU without peer access) is
 *            refused with LVSA_ERR_INVALID_ARG before any launch.
 *   chunk_tokens  HOST int array of nchunks token counts (>= 0, sum >= 1);
 *            ranges follow one another in array order.
 *   nchunks  1..64.   heads, head0, band: 0 <= head0, 1 <= band,
 *            head0 + band <= heads.   d: 64 or 128.   batch: 1..21845.
 *   q_band, k_band, v_band  DEVICE bf16 [batch][sum of chunk_tokens][band][d],
 *            16-byte aligned, pairwise disjoint and disjoint from every local
 *            range buffer.
 *   stream   a cudaStream_t (as void*).
 * Behaviour: asynchronous; one launch for the three tensors.  The caller makes
 * sure the range buffers are written (and not rewritten) while it runs.
 */
lvsa_status lvsa_seq_to_heads(const void* const* q_chunks, const void* const* k_chunks,
                              const void* const* v_chunks, const int* chunk_tokens, int nchunks,
                              int heads, int head0, int band, int d, int batch,
                              void* q_band, void* k_band, void* v_band, void* stream);

/*
 * lvsa_attention_to_chunks -- lvsa_attention over a band of heads whose output
 * rows go to token-range buffers: row i of the sequence is stored into the
 * buffer c with start_c <= i < start_c + chunk_tokens[c], at token i - start_c
 * and head head0 + h of its rows of out_heads heads.  The same arithmetic as
 * lvsa_attention: the stored values are bit for bit those lvsa_attention
 * writes for the same heads.
 *
 * Arguments:
 *   q, k, v, lists, L, T, tokens_per_frame, heads, d, batch, scale  as
 *            lvsa_attention (q, k, v: [batch][T*P][heads][d], e.g. the band
 *            buffers of lvsa_seq_to_heads).
 *   out_chunks  HOST array of nchunks pointers addressable from this GPU (its
 *            memory, another GPU's with peer access -- enabled here if it is
 *            not yet -- a peer mapping, or pinned host memory), buffer c =
 *            [batch][chunk_tokens[c]][out_heads][d] bf16, 16-byte aligned,
 *            disjoint from each other, from q, k, v and from lists; may be NULL
 *            where chunk_tokens[c] == 0.  Memory CUDA does not know, or knows
 *            but cannot address from the GPU (pageable host memory, another
 *            GPU without peer access), is refused (LVSA_ERR_INVALID_ARG).
 *            Heads outside [head0, head0 + heads) are not written.
 *   chunk_tokens  HOST int array, >= 0 each, summing to T * tokens_per_frame.
 *   nchunks  1..64.   out_heads, head0: head0 >= 0, head0 + heads <= out_heads.
 *   stream   a cudaStream_t (as void*).
 * Behaviour: asynchronous; errors as lvsa_attention.  When a buffer is not
 * this GPU's memory the kernel releases its stores at system scope before it
 * ends, so the owner sees them once it has synchronised with this rank after
 * the kernel (stream synchronisation, then a barrier).
 */
lvsa_status lvsa_attention_to_chunks(const void* q, const void* k, const void* v,
                                     const int32_t* lists, int L, int T, int tokens_per_frame,
                                     int heads, int d, int batch, float scale,
                                     void* const* out_chunks, const int* chunk_tokens, int nchunks,
                                     int out_heads, int head0, void* stream);

/* Bytes of an IPC handle written by lvsa_ipc_export. */
#define LVSA_IPC_HANDLE_BYTES 72

/*
 * lvsa_ipc_export -- writes an LVSA_IPC_HANDLE_BYTES handle for the device
 * buffer holding dev_ptr (a CUDA IPC handle of its allocation plus the offset
 * of dev_ptr in it) into the HOST buffer `handle`, for another process to map.
 * dev_ptr must come from cudaMalloc (directly or through a caching allocator
 * that uses it); memory from the virtual-memory API cannot be exported this
 * way (LVSA_ERR_CUDA).  Errors: LVSA_ERR_INVALID_ARG (NULL, not device memory).
 */
lvsa_status lvsa_ipc_export(const void* dev_ptr, void* handle);

/*
 * lvsa_ipc_import -- maps the buffer of a handle written by lvsa_ipc_export in
 * ANOTHER process (the same process cannot map its own handles) into this
 * process on the current device, with peer access enabled when the buffer is
 * on another GPU, and returns the pointer to use in *dev_ptr.  Mappings of the
 * same allocation are shared and counted; release each pointer once.
 */
lvsa_status lvsa_ipc_import(const void* handle, void** dev_ptr);

/* lvsa_ipc_release -- drops a pointer returned by lvsa_ipc_import (the mapping
 * is closed with the last pointer into it).  LVSA_ERR_INVALID_ARG for a pointer
 * that lvsa_ipc_import did not return or that was already released. */
lvsa_status lvsa_ipc_release(void* dev_ptr);

/*
 * lvsa_get_device_status -- device status bits (LVSA_DEV_*) of the current
 * device, OR-ed over every kernel since the last clear.  Synchronises the
 * device.  clear != 0 resets them to 0 afterwards.
 */
lvsa_status lvsa_get_device_status(unsigned int* flags, int clear);

/*
 * lvsa_set_wait_budget_ns -- time budget of every device-side wait of later
 * launches (default 4e9 ns, counted in SM cycles at 2 cycles per ns).  Values
 * below 1000 ns are raised to 1000 ns; values above 1e12 ns (1000 s) are
 * refused with LVSA_ERR_INVALID_ARG and the budget is left unchanged.
 */
lvsa_status lvsa_set_wait_budget_ns(unsigned long long ns);

/*
 * lvsa_watchdog_selftest -- launches one CTA that waits on a barrier nobody
 * arrives on, with the given budget, through the same bounded-wait code the
 * attention kernel uses.  The wait runs out, sets LVSA_DEV_TIMEOUT and the
 * kernel returns normally (no trap, no fault).  Used to test failure detection.
 */
lvsa_status lvsa_watchdog_selftest(unsigned long long budget_ns, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* lvsa_status_string(int status);

/* Library ABI version (major*10000 + minor*100 + patch). */
int lvsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LVSA_H */
