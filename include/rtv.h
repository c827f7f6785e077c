/*
 * rtv.h -- C ABI of librtv: per-chunk KV-cache upkeep and FP8 attention for
 * batch-size-one autoregressive video diffusion serving, on one B200 (sm_100a).
 *
 * What the library computes (sources are the pages' titles and sections):
 *   - aidose.in, "Runway explains how it serves a 57B video model in real
 *     time", third paragraph: rotary position embedding and FP8
 *     quantisation are applied a single time, as each frame is written into
 *     the KV cache; the cache is a ring buffer whose advance copies nothing;
 *     attention then runs over the cached frames.
 *   - pttl.gr, section "Από οκτώ H100 σε τέσσερις", second paragraph: the
 *     same write-time transformation and circular buffer; 240 attention calls
 *     per diffusion step.
 * The pages do not give the RoPE layout, the FP8 format, the scale
 * granularity, the window or the mask.  This library implements: 3D axial
 * rotate-half RoPE over (frame t, grid row h, grid column w) segments of
 * head_dim, base rope_base, angles in fp64; OCP E4M3 codes with one fp32
 * scale amax/448 per (token, head) for Q, K and V (an item whose amax is
 * below 2^-119, where the fp32 reciprocal 448/amax would overflow, is stored
 * as zero -- zero codes, scale 0 -- like an all-zero item); a ring of
 * window_frames + max_frames_per_chunk slots plus an optional pinned slot;
 * softmax(q.k / sqrt(head_dim)) attention of the chunk's queries over the
 * pinned frame, the window and the chunk's own frames, with no mask inside
 * that key set (bidirectional within the chunk).
 *
 * Conventions for every call:
 *   - Pointers named q/k/v/out/device_buf are DEVICE pointers on the device
 *     that was current when the cache was created; the stream argument is a
 *     cudaStream_t passed as void* (NULL = legacy default stream).
 *   - Calls validate their arguments on the host before launching and return
 *     a status; they never abort and never throw.
 *   - rtv_cache_append, rtv_attend and rtv_cache_advance never synchronise
 *     the host with the device: all device work is stream-ordered.
 *   - A cache object is not thread-safe: one host thread drives it.
 */
#ifndef RTV_H
#define RTV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RTV_OK = 0,
    RTV_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment, layer or frame count */
    RTV_ERR_OOM = 2,         /* device allocation failed, or caller buffer too small */
    RTV_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
    RTV_ERR_STATE = 4,       /* call not valid in the cache's current state */
    RTV_ERR_TIMEOUT = 5,     /* a kernel's bounded wait ran out (see rtv_poll_error) */
    RTV_ERR_UNSUPPORTED = 6, /* configuration outside what the kernels implement */
    RTV_ERR_BOUNDS = 7       /* a debug build's kernel found a slot index out of range */
} rtv_status;

/* Output element types of rtv_attend. */
enum { RTV_OUT_F32 = 0, RTV_OUT_BF16 = 1 };

/* Largest number of slots (pinned + ring) a cache may have. */
#define RTV_MAX_SLOTS 64
/* Largest number of frames one chunk may stage. */
#define RTV_MAX_FRAMES_PER_CHUNK 4

typedef struct rtv_cache rtv_cache;

/*
 * Cache configuration.
 *   n_layers              layers, each with its own K/V ring and Q workspace
 *   n_heads, head_dim     attention heads and per-head width; head_dim is 64
 *                         or 128
 *   grid_h, grid_w        latent grid of one frame; T = grid_h * grid_w
 *                         tokens per frame, token k at row k / grid_w and
 *                         column k % grid_w (row-major)
 *   max_frames_per_chunk  F_max, 1..RTV_MAX_FRAMES_PER_CHUNK
 *   window_frames         W >= 0 committed frames kept visible
 *   pinned_frames         0 or 1; with 1, the first chunk (one frame, the
 *                         conditioning frame at absolute index 0) is kept in
 *                         slot 0 for the life of the cache
 *   rope_t, rope_h, rope_w  RoPE segment widths along head_dim, in the order
 *                         t | h | w; they sum to head_dim and each half-width
 *                         (rope_x / 2) is a multiple of head_dim / 16
 *   rope_base             RoPE base (10000 in the workloads)
 * Slots: P0 = pinned_frames, C = W + F_max ring slots, P0 + C <= RTV_MAX_SLOTS.
 */
typedef struct {
    int n_layers;
    int n_heads;
    int head_dim;
    int grid_h;
    int grid_w;
    int max_frames_per_chunk;
    int window_frames;
    int pinned_frames;
    int rope_t;
    int rope_h;
    int rope_w;
    double rope_base;
} rtv_cache_config;

/*
 * Ring state, as the host bookkeeping holds it.
 *   frames_committed     absolute index of the next frame to be staged
 *                        (pinned frame, if committed, plus generated frames)
 *   generated_committed  G: generated frames committed
 *   pinned_committed     1 once the pinned conditioning frame is committed
 *   head                 slot of the next generated frame: P0 + (G mod C)
 *   n_visible            committed frames attention sees: pinned + min(G, W)
 *   visible_slots/frames the visible frames in logical order (pinned, then
 *                        oldest to newest) with their slots
 *   frame_of_slot        per slot, the visible frame it holds, or -1
 *   staged_layers        layers that currently hold staged frames
 *   staged_frames        their frame count (-1 if the layers disagree)
 *   last_attend_splits   key-range splits of the last rtv_attend call (0
 *                        before the first): 1 = one kernel, s > 1 = the
 *                        attention kernel over s key ranges plus a merge
 *                        kernel
 */
typedef struct {
    long long frames_committed;
    long long generated_committed;
    int pinned_committed;
    int head;
    int n_slots;
    int n_visible;
    int visible_slots[RTV_MAX_SLOTS];
    long long visible_frames[RTV_MAX_SLOTS];
    long long frame_of_slot[RTV_MAX_SLOTS];
    int staged_layers;
    int staged_frames;
    int last_attend_splits;
} rtv_cache_state;

/*
 * Byte offsets, inside the cache's device buffer, of one layer's tensors.
 *   k_codes, v_codes  uint8 E4M3 [n_slots][n_heads][T][head_dim]
 *   k_scales, v_scales fp32 [n_slots][n_heads][scale_pitch]   (first T used)
 *   q_codes           uint8 E4M3 [n_heads][F_max * T][head_dim]
 *   q_scales          fp32 [n_heads][q_scale_pitch]           (first F_max*T used)
 *   v_scale_max       uint64 [n_slots][n_heads]: (append sequence << 32) |
 *                     fp32 bits of the largest V scale of that frame and head
 */
typedef struct {
    size_t k_codes, v_codes, k_scales, v_scales, q_codes, q_scales, v_scale_max;
    int scale_pitch;
    int q_scale_pitch;
} rtv_layer_layout;

/* Human-readable name of a status (static storage; never NULL). */
const char* rtv_status_string(rtv_status status);

/*
 * Device bytes a cache with this configuration needs (K/V rings, scales, Q
 * workspaces, RoPE tables, the key-range split partials of one attention
 * call -- 4 x F_max*T x n_heads x (head_dim + 2) fp32, shared by all layers --
 * and the error word), so that a caller can allocate them itself.  Errors: RTV_ERR_INVALID_ARG (NULL or inconsistent config),
 * RTV_ERR_UNSUPPORTED (head_dim or RoPE split the kernels do not implement).
 */
rtv_status rtv_cache_required_bytes(const rtv_cache_config* cfg, size_t* bytes);

/* Offsets of one layer's tensors in the device buffer (see rtv_layer_layout). */
rtv_status rtv_cache_layer_layout(const rtv_cache_config* cfg, int layer, rtv_layer_layout* out);

/*
 * Create a cache on the current CUDA device.  device_buf: NULL to let the
 * library cudaMalloc (and later free) the buffer, or a caller-owned device
 * buffer of at least rtv_cache_required_bytes bytes, 256-byte aligned, which
 * the caller keeps alive until rtv_cache_destroy returns.  The buffer is
 * zeroed (synchronously) and the RoPE h/w tables are uploaded.
 * Errors: RTV_ERR_INVALID_ARG, RTV_ERR_UNSUPPORTED, RTV_ERR_OOM, RTV_ERR_CUDA.
 */
rtv_status rtv_cache_create(const rtv_cache_config* cfg, void* device_buf, size_t buf_bytes,
                            rtv_cache** out);

/* Destroy a cache (synchronises the device; frees what the library owns). */
rtv_status rtv_cache_destroy(rtv_cache* cache);

/*
 * Stage a chunk of n_frames frames for one layer: one fused kernel applies
 * 3D RoPE to Q and K, computes each (token, head) row's amax and scale, and
 * writes E4M3 codes and fp32 scales -- K and V into the ring slots of the
 * staged frames, Q into the layer's Q workspace.
 * Source: aidose.in, "Runway explains how it serves a 57B video model in real
 * time", third paragraph (rotary embedding and FP8 quantisation are applied
 * once, when a frame is written into the cache); pttl.gr, section "Από οκτώ
 * H100 σε τέσσερις", second paragraph (the same write-time transformation).
 *   q, k, v   bf16 [n_frames * T][n_heads][head_dim], row-major (the hidden
 *             dimension n_heads*head_dim contiguous), 16-byte aligned, not
 *             modified; read once.  Owned by the caller; only read while the
 *             launched kernel runs (stream-ordered).
 *   n_frames  1..max_frames_per_chunk (exactly 1 for the pinned chunk).
 * Absolute frame index of staged frame f = frames_committed + f.  Appending
 * again to the same layer before rtv_cache_advance overwrites its staged
 * frames (several denoising passes per chunk).  The library cannot check the
 * sizes of q/k/v: the caller passes n_frames*T*n_heads*head_dim elements each.
 * Errors: RTV_ERR_INVALID_ARG (layer, n_frames, NULL or misaligned pointer),
 * RTV_ERR_STATE (layers staged with different frame counts), RTV_ERR_CUDA.
 */
rtv_status rtv_cache_append(rtv_cache* cache, int layer, const void* q, const void* k,
                            const void* v, int n_frames, void* stream);

/*
 * The QKV projection with the append fused into it: an FP8 GEMM on tcgen05
 * tensor cores whose epilogue does rtv_cache_append's work on the projected
 * Q/K/V, so the bf16 Q/K/V are never written to or read from memory.
 * Source: lhc.media, "Runway partage la construction de Runway Characters",
 * third paragraph (matmul and kernel tuning); aidose.in, "Runway explains how
 * it serves a 57B video model in real time", third paragraph (FP8 matmuls;
 * rotary embedding and FP8 quantisation applied once, at cache write).
 *   x_codes   E4M3 [n_frames*T][hidden] activations, row-major, 16-byte aligned
 *   x_scales  fp32 [n_frames*T], one per token row
 *   w_codes   E4M3 [3*n_heads*head_dim][hidden] weights, row-major (one output
 *             feature per row: the Q heads, then the K heads, then the V
 *             heads, each head's head_dim features contiguous), 16-byte aligned
 *   w_scales  fp32 [3*n_heads*head_dim], one per output feature, 16-byte aligned
 *   hidden    a multiple of 128
 * The projected value of row r, feature n is
 *     bf16( fl( fl(acc * x_scales[r]) * w_scales[n] ) ),
 *     acc = sum_k decode(x_codes[r][k]) * decode(w_codes[n][k]) (fp32),
 * and the cache then receives exactly what rtv_cache_append would write for
 * that bf16 Q/K/V (same staging, overwrite and frame rules).  Supported for
 * head_dim 128 with the RoPE split 32:48:48 and an even n_heads.
 * Errors: as rtv_cache_append, plus RTV_ERR_UNSUPPORTED (other shapes).
 */
rtv_status rtv_cache_append_project(rtv_cache* cache, int layer, const void* x_codes,
                                    const float* x_scales, const void* w_codes,
                                    const float* w_scales, int hidden, int n_frames, void* stream);

/*
 * Attention of the layer's staged chunk over its key set (pinned frame,
 * window oldest to newest, staged frames).
 * Source: aidose.in, "Runway explains how it serves a 57B video model in real
 * time", third paragraph (attention runs over the cache whose frames were
 * rotated and quantised at write time); pttl.gr, section "Από οκτώ H100 σε
 * τέσσερις", second paragraph (240 attention calls per diffusion step).
 * The result is written to
 *   out  [n_frames * T][n_heads][head_dim], fp32 (RTV_OUT_F32) or bf16
 *        (RTV_OUT_BF16), row-major, 16-byte aligned.
 * One kernel: TMA loads of Q/K/V codes and scales by (slot, head, token
 * tile) coordinates, QK^T in FP8 E4M3 on tcgen05 tensor cores into TMEM,
 * online softmax in registers, PV on tcgen05 with P and the V codes in f16.
 * When one CTA per (head, 256 query rows) would leave the GPU's last wave of
 * CTAs mostly idle, the key set is split into up to 4 ranges (grid z): each
 * CTA writes its range's unnormalised O and row statistics to the cache
 * buffer's split section and a second kernel merges them (online-softmax
 * merge) into out.  That section is shared by all layers: attention calls on
 * one cache must be ordered on one stream (as the append/attend/advance
 * sequence already is); overlapping calls race.
 * Errors: RTV_ERR_INVALID_ARG, RTV_ERR_STATE (layer has no staged frames),
 * RTV_ERR_CUDA.  A kernel timeout is reported by rtv_poll_error.
 */
rtv_status rtv_attend(rtv_cache* cache, int layer, void* out, int out_dtype, void* stream);

/*
 * Commit the staged frames of every layer (host bookkeeping only; launches
 * nothing and copies nothing).  Requires all layers staged with the same
 * frame count.  Source: aidose.in, "Runway explains how it serves a 57B video
 * model in real time", third paragraph (the cache is a ring buffer that moves
 * forward without copying); pttl.gr, section "Από οκτώ H100 σε τέσσερις",
 * second paragraph (circular buffer).  Errors: RTV_ERR_STATE.
 */
rtv_status rtv_cache_advance(rtv_cache* cache);

/*
 * Whole-step CUDA graph with the ring state resident on the device.
 * Source: lhc.media, "Runway partage la construction de Runway Characters",
 * third paragraph (CUDA graphs among the serving optimisations); aidose.in,
 * "Runway explains how it serves a 57B video model in real time", fourth
 * paragraph (one host synchronisation per step cost 168.5 -> 278 ms): the
 * host should only launch, never wait, and launch as little as possible.
 *
 * rtv_step_graph_create captures one steady-state step of every layer --
 * rtv_cache_append then rtv_attend for layers 0..n_layers-1, then a one-warp
 * kernel that advances the ring state held in the cache buffer -- into one
 * CUDA graph.  The captured kernels read the staged and key-set slots, the
 * frame-axis RoPE cos/sin and the V-scale tag from that device state instead
 * of their launch parameters, so the same graph serves every later step.
 *   n_frames      frames per chunk, 1..max_frames_per_chunk
 *   q, k, v       arrays of n_layers device pointers: each layer's bf16
 *                 [n_frames*T][n_heads][head_dim] inputs; the graph reads
 *                 whatever these buffers hold when it runs, so the caller
 *                 writes each step's Q/K/V into them (stream-ordered) before
 *                 rtv_step_graph_launch
 *   out           array of n_layers device pointers, each layer's output as
 *                 for rtv_attend (out_dtype RTV_OUT_F32 or RTV_OUT_BF16)
 *   stream        a non-NULL stream: used for the capture (legacy-stream
 *                 capture is not allowed); synchronised once
 * Requires the steady state: the pinned frame committed (when configured),
 * at least window_frames generated frames committed, no layer staged.  The
 * caller keeps the buffers alive until rtv_step_graph_destroy.
 * Errors: RTV_ERR_INVALID_ARG, RTV_ERR_STATE (not steady), RTV_ERR_CUDA,
 * RTV_ERR_OOM.
 *
 * rtv_step_graph_launch enqueues one step on `stream` (no host
 * synchronisation) and makes the same step in the host ring state (as
 * rtv_cache_advance would after every layer's append), so rtv_cache_get_state
 * and direct calls stay consistent.  Direct append/attend/advance calls may
 * be mixed in between: if they moved the ring, the launch first copies the
 * current state to the device (stream-ordered).  Errors: RTV_ERR_INVALID_ARG,
 * RTV_ERR_STATE (a layer is staged by a direct call), RTV_ERR_CUDA.
 */
typedef struct rtv_step_graph rtv_step_graph;
rtv_status rtv_step_graph_create(rtv_cache* cache, int n_frames, const void* const* q,
                                 const void* const* k, const void* const* v, void* const* out,
                                 int out_dtype, void* stream, rtv_step_graph** graph);
rtv_status rtv_step_graph_launch(rtv_step_graph* graph, void* stream);
rtv_status rtv_step_graph_destroy(rtv_step_graph* graph);

/* Ring state (host-side; no device access). */
rtv_status rtv_cache_get_state(const rtv_cache* cache, rtv_cache_state* out);

/* Device pointer of the cache buffer and its size. */
rtv_status rtv_cache_device_buffer(const rtv_cache* cache, void** ptr, size_t* bytes);

/*
 * Copy one slot of one layer, and the layer's Q workspace, to HOST buffers
 * (test and debug use; waits for the stream).
 *   codes_k, codes_v  [n_heads][T][head_dim] bytes of the slot
 *   sk, sv            [n_heads][T] floats of the slot
 *   q_codes           [n_heads][max_frames_per_chunk * T][head_dim] bytes
 *   sq                [n_heads][max_frames_per_chunk * T] floats
 * (the Q workspace rows of the staged frames come first).  Any pointer may be
 * NULL to skip that tensor.  Errors: RTV_ERR_INVALID_ARG (layer, slot),
 * RTV_ERR_CUDA.
 */
rtv_status rtv_cache_export(const rtv_cache* cache, int layer, int slot, void* codes_k,
                            void* codes_v, float* sk, float* sv, void* q_codes, float* sq,
                            void* stream);

/*
 * Read (and clear) the device error word.  Synchronises the device; the only
 * call that does.  Returns RTV_ERR_TIMEOUT if a kernel's bounded wait ran
 * out since the last poll, RTV_OK otherwise.
 */
rtv_status rtv_poll_error(rtv_cache* cache);

/*
 * The key-range split rtv_attend chooses (host arithmetic only; no device
 * needed).  n_units = ceil(n_frames*T / 256) * n_heads CTAs of one key range
 * each, n_kv_tiles = key frames * ceil(T / 64), sm_count = the device's SMs.
 * Out: n_split in 1..4 and tiles_per_split (the last split may hold fewer,
 * none is empty).  The plan minimises ceil(n_units*s / sm_count) / s plus 3%
 * per extra split, with at least 8 KV tiles per split.
 * Errors: RTV_ERR_INVALID_ARG (a count < 1 or a NULL output).
 */
rtv_status rtv_split_plan(int n_units, int n_kv_tiles, int sm_count, int* n_split,
                          int* tiles_per_split);

/*
 * rtv_attend for callers that cannot allocate device memory: the same
 * kernels and results (bit for bit), but the key-range split partials go to a
 * fixed 16 MiB device array compiled into the library (file-scope
 * __device__) instead of the cache buffer's split section.  The call
 * allocates nothing (no cudaMalloc/cudaFree, no allocating library routine).
 * Device footprint: every device on which a cache is created holds the
 * 16 MiB array until the process exits -- rtv_cache_create looks up its
 * address (once per device, with that device current), which makes the
 * CUDA runtime load the module that holds it; if that lookup failed there,
 * the first call of this entry point retries it.  Nothing in the array needs
 * to start at zero: the merge reads only partials the same call wrote.  The
 * array is shared by every cache and stream on the device: calls that
 * overlap in time (other streams, other host threads) race.  A call whose
 * split plan needs more than 16 MiB of partials (n_split x n_frames*T x
 * n_heads x (head_dim + 2) fp32) is rejected with RTV_ERR_UNSUPPORTED before
 * anything is launched; an unsplit call needs none.  The method's sources
 * describe no counterpart of this entry point: it is a deployment
 * convenience.
 * Errors: as rtv_attend, plus RTV_ERR_UNSUPPORTED (partials over 16 MiB) and
 * RTV_ERR_CUDA (symbol lookup failed).
 */
rtv_status rtv_attend_static_scratch(rtv_cache* cache, int layer, void* out, int out_dtype,
                                     void* stream);

/*
 * Test hook: when set to 1, the next rtv_attend launches the kernel in a mode
 * where its first wait can never complete (the producer never arms the
 * barrier and issues no copy), so every wait runs into its time limit, the
 * kernel records RTV_ERR_TIMEOUT in the error word and returns cleanly.
 * wait_limit_cycles sets the per-wait limit in SM clock cycles (0 = default,
 * about one second).  Used only by the failure-detection test.
 */
rtv_status rtv_debug_set_wait_fault(rtv_cache* cache, int enable, long long wait_limit_cycles);

/*
 * Debug builds (librtv_debug.so, compiled with RTV_DEBUG): every kernel
 * checks the ring slots it is given against the cache's slot count before it
 * touches memory; a launch that finds one out of range records it in the
 * device error word and returns, and rtv_poll_error then reports
 * RTV_ERR_BOUNDS.  rtv_debug_build returns 1 in such a build, 0 otherwise.
 * rtv_debug_corrupt_next_attend makes the next rtv_attend name slot
 * `bad_slot` first in its key set (the test of that check); it returns
 * RTV_ERR_UNSUPPORTED in a release build, where nothing would catch it.
 */
int rtv_debug_build(void);
rtv_status rtv_debug_corrupt_next_attend(rtv_cache* cache, int bad_slot);

#ifdef __cplusplus
}
#endif

#endif /* RTV_H */
