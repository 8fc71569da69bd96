/*
 * fmoe.h -- C ABI of the quantised mixture-of-experts decode library for
 * NVIDIA B200 (sm_100a).
 *
 * One call runs one mixture-of-experts layer of the decode step that the
 * Flash-MoE pages describe.  The Hysen Labs page "Flash-MoE: Running a 397B
 * Parameter Model on a Laptop", section "How the SSD expert streaming pipeline
 * works", splits it over a GPU command buffer (normalisation, routing GEMV,
 * shared expert), the host (softmax and top-K) and a second command buffer
 * (the routed experts and the combine).  The themata summary of the same title
 * (Key Takeaways) gives 512 experts per layer with K = 4 active; "Flash-MoE:
 * Running a 400 Billion Parameter Model on a MacBook", section "The
 * Architecture", sizes a 4-bit expert at about 6.75 MB and dequantises it with
 * fused multiply-adds.
 * Here every step runs on the GPU and all expert weights stay resident in HBM.
 *
 * Conventions for every entry point
 *  - Pointers named *_dev are device pointers the caller allocates and owns
 *    (the library only borrows them); they must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls other than fmoe_create / fmoe_destroy / fmoe_poll_status only
 *    enqueue work on `stream` and never synchronise the host.  Calls on one
 *    context share its device workspace, so they must be ordered on one stream.
 *  - bf16 tensors are raw bf16 bit patterns (uint16 storage).
 *  - Every call validates its arguments before touching the GPU and returns an
 *    fmoe_status; fmoe_last_error() gives a one-line reason.  CUDA launch
 *    errors are reported as FMOE_ERR_CUDA.
 */
#ifndef FMOE_H
#define FMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FMOE_API __attribute__((visibility("default")))
#else
#define FMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct fmoe_ctx fmoe_ctx;

typedef enum fmoe_status {
  FMOE_OK = 0,
  FMOE_ERR_INVALID_ARG = 1, /* bad value, NULL pointer, unknown/destroyed context */
  FMOE_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement     */
  FMOE_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned                  */
  FMOE_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed               */
  FMOE_ERR_OOM = 5,         /* device allocation failed                           */
  FMOE_ERR_TIMEOUT = 6      /* a device-side bounded wait ran out (fmoe_poll_status) */
} fmoe_status;

/* fmoe_config.flags */
#define FMOE_FLAG_FORCE_PER_TOKEN 0x1u /* T > 1: run the batch-1 kernel once per token  */
#define FMOE_FLAG_FORCE_GROUPED 0x2u   /* T >= 1: always use the grouped batched path   */
/* fmoe_stack_forward on the batch-1 kernel: one launch per layer and token
 * instead of one launch per token running every layer of the range. */
#define FMOE_FLAG_STACK_PER_LAYER 0x4u
/* The grouped batched path needs n_experts <= 1023 and max_tokens <= 16320:
 * beyond either a context runs every token count through the batch-1 kernel,
 * and FORCE_GROUPED makes fmoe_create fail with FMOE_ERR_UNSUPPORTED. */
/* Fault injection for tests: the router step never publishes its completion,
 * so every block's bounded wait for it runs out and the call reports
 * FMOE_ERR_TIMEOUT through fmoe_poll_status (no GPU fault, no hang). */
#define FMOE_FLAG_DEBUG_SKIP_ROUTER_RELEASE 0x100u

typedef struct fmoe_config {
  int32_t hidden;      /* H: model width; multiple of 64, at most 4096          */
  int32_t n_experts;   /* E: routed experts per layer (>= 1)                      */
  int32_t top_k;       /* K: experts selected per token, 1 <= K <= min(E, 8)     */
  int32_t inter;       /* I: SwiGLU intermediate width; multiple of 64, <= 4096  */
  int32_t bits;        /* code width of expert weights: 4 or 2                    */
  int32_t group;       /* quantisation group along the input dimension: must be 64 */
  int32_t n_layers;    /* number of layer descriptors passed to fmoe_create      */
  int32_t max_tokens;  /* largest T any call will pass (0 means 256)             */
  float rms_eps;       /* RMSNorm epsilon (used by layers with norm_w != NULL)   */
  uint32_t flags;      /* FMOE_FLAG_*                                             */
  uint32_t wait_timeout_us; /* device-side bounded-wait limit; 0 means 1 second */
} fmoe_config;

/* Per-layer weights, all device pointers owned by the caller. */
typedef struct fmoe_layer_desc {
  const void* router_w_dev;    /* bf16 [E][H] row-major router GEMV weight            */
  const float* router_bias_dev;/* fp32 [E] added to the logits, or NULL              */
  void* experts_dev;           /* E routed + 1 shared expert blobs, contiguous: blob e
                                  at byte offset e * fmoe_expert_bytes(H, I, bits), the
                                  shared expert last (index E).  Given in the canonical
                                  format below; fmoe_create rewrites it IN PLACE into
                                  the library's packed tile layout (same size), and it
                                  must stay allocated and unmodified until destroy.   */
  const void* norm_w_dev;      /* bf16 [H] RMSNorm weight applied to the layer input
                                  before routing and experts, or NULL for no norm.    */
} fmoe_layer_desc;

/*
 * Canonical expert blob (input format of fmoe_create; output of
 * fmoe_unpack_expert).  For each matrix in order gate [I][H], up [I][H],
 * down [H][I] (rows x input columns):
 *   codes : R*C*bits/8 bytes, row-major, 32/bits codes per little-endian
 *           uint32; code c of a row is at bit bits*(c % (32/bits)) of word
 *           c / (32/bits) of that row;
 *   scales: bf16 [R][C/64];  biases: bf16 [R][C/64];
 * weight w[r][c] = scale[r][c/64] * code[r][c] + bias[r][c/64].
 * At H = 4096, I = 1024 a blob is 7,077,888 bytes at 4 bits (the pages size an
 * expert at about 6.75 MB) and 3,932,160 bytes at 2 bits.
 */
FMOE_API size_t fmoe_expert_bytes(int32_t hidden, int32_t inter, int32_t bits);

/*
 * Creates a context on the current CUDA device: validates `cfg` and the layer
 * descriptors (copied; the weights they point to are borrowed), allocates the
 * device workspace, and repacks every layer's experts_dev in place from the
 * canonical to the packed layout on `stream` (then synchronises it).
 * Both paths apply the bf16 scale and bias in fp32 to exact integer codes, so
 * any bf16 value is taken as it is.
 * Errors: INVALID_ARG (NULL, bad shapes, K > E, bits not 2/4, group != 64),
 * UNSUPPORTED (H or I above 4096 or a shape whose shared-memory plan does not
 * fit), ALIGNMENT, OOM, CUDA.  On error *out is NULL.
 */
FMOE_API fmoe_status fmoe_create(const fmoe_config* cfg, const fmoe_layer_desc* layers, void* stream, fmoe_ctx** out);

/*
 * Passage: the Hysen Labs page "Flash-MoE: Running a 397B Parameter Model on
 * a Laptop", section "How the SSD expert streaming pipeline works": only the
 * K = 4 selected experts of a layer are read from storage, and the operating
 * system's page cache (standard LRU, about 35 GB) serves roughly 71% of them.
 * Here host memory plays the storage and an HBM pool of expert slots the page
 * cache.
 * As fmoe_create, except that every layers[l].experts_dev is a HOST pointer to
 * page-locked memory (cudaHostAlloc, or cudaHostRegister with mapping)
 * holding the layer's E + 1 canonical blobs; it is repacked in place (it must
 * stay allocated and unmodified until destroy).  The shared experts are copied
 * into HBM; the routed experts stay in host memory behind a cache of
 * `cache_slots` expert slots in HBM (2 * top_k <= cache_slots; more than
 * n_layers * n_experts are not used), shared by all layers.  The fused kernel
 * consults the cache after routing: a hit is read from its slot; a miss is
 * read from host memory over the host link and, as its tiles arrive, written
 * into a slot chosen by CLOCK replacement (second chance, the textbook
 * approximation of LRU), all in the same launch, so no host round trip is
 * involved.  Results are bit-identical to a resident context's.  Such a
 * context runs every call on the batch-1 kernel, one launch per layer and
 * token; fmoe_expert_forward returns UNSUPPORTED.  Calls on one cached context
 * must be ordered on one stream (the cache state is part of the context).
 * Errors: as fmoe_create; INVALID_ARG also for cache_slots < 2 * top_k or
 * experts that are not page-locked host memory.
 */
FMOE_API fmoe_status fmoe_create_cached(const fmoe_config* cfg, const fmoe_layer_desc* layers, int64_t cache_slots,
                                        void* stream, fmoe_ctx** out);

/* Synchronises `stream` and returns the expert-cache hit and miss counts of a
 * cached context since create (each routed pick of each launch counts once).
 * Errors: INVALID_ARG (no cache), CUDA. */
FMOE_API fmoe_status fmoe_cache_stats(fmoe_ctx* ctx, void* stream, uint64_t* hits, uint64_t* misses);

/*
 * Passage: the Hysen Labs page "Flash-MoE: Running a 397B Parameter Model on
 * a Laptop", section "How the SSD expert streaming pipeline works": the second
 * command buffer normalises the layer input and computes the routing logits,
 * then the host takes a softmax and the top K; the themata summary of the same
 * title (Key Takeaways) gives 512 experts per layer with K = 4.
 * Router step of layer `layer` for T tokens: z = RMSNorm(x) when the layer has
 * a norm weight (else z = x), logits = W_r z (+ bias) in fp32, softmax, the K
 * largest probabilities in descending order (equal values: lower expert index
 * first) and their renormalised weights w_k = p_k / sum_j p_j.  A NaN logit
 * counts as -inf; when the largest logit is infinite the softmax is taken as
 * its limit, so the picks equal to it share the weight equally (each of K
 * picks gets 1/K when every logit is -inf).
 *   x_dev   : bf16 [T][H];  idx_dev : int32 [T][K];  w_dev : fp32 [T][K].
 * T == 0 is a no-op.  Errors: INVALID_ARG (layer or T out of range, NULL),
 * ALIGNMENT, CUDA.
 */
FMOE_API fmoe_status fmoe_route(fmoe_ctx* ctx, int32_t layer, const void* x_dev, int32_t T, int32_t* idx_dev,
                       float* w_dev, void* stream);

/*
 * The router step of fmoe_route (same inputs, outputs and selection rule)
 * computed without any device allocation: its only scratch, the fp32 logits
 * [T][E], is a fixed 128 KB device array inside the library.  The pages have
 * no counterpart; it exists for callers that cannot allocate device memory per
 * call -- a loop whose device memory is held entirely by its own pool
 * allocator, or one that cannot take cudaFree's device-wide synchronisation.
 * Limits: T * E <= 32768 and T <= 4096; larger calls return UNSUPPORTED
 * before any GPU work.  fmoe_create looks up the array's address on its
 * device (cudaGetSymbolAddress), so calls on a context never do, and may be
 * captured into a CUDA graph; a call on a device where no context was created
 * made inside a stream capture returns UNSUPPORTED instead of looking it up.
 * Calls that overlap in time share the array and race: order them on one
 * stream.  Weights follow fmoe_route's rule, including its limit for an
 * infinite largest logit.
 * Logits accumulate in a different order than fmoe_route's, so weights may
 * differ in the last bits; the indices agree except at near-ties.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED, CUDA.
 */
FMOE_API fmoe_status fmoe_route_static(fmoe_ctx* ctx, int32_t layer, const void* x_dev, int32_t T,
                                       int32_t* idx_dev, float* w_dev, void* stream);

/*
 * Passage: "Flash-MoE: Running a 400 Billion Parameter Model on a MacBook",
 * section "The Architecture" (each active expert's weights dequantised inside
 * fused multiply-adds, about 6.75 MB per expert at 4 bits), and the Hysen Labs
 * page's section "How the SSD expert streaming pipeline works" (the third
 * command buffer runs the expert forward pass).
 * One expert's SwiGLU feed-forward on the layer's (normed) input:
 * y = W_down (silu(W_gate z) * (W_up z)), z as in fmoe_route.
 *   expert  : 0..E-1 for a routed expert, -1 for the shared expert.
 *   x_dev   : bf16 [T][H];  y_dev : fp32 [T][H].
 * T == 0 is a no-op.  Errors: INVALID_ARG (expert, layer or T out of range),
 * ALIGNMENT, CUDA.
 */
FMOE_API fmoe_status fmoe_expert_forward(fmoe_ctx* ctx, int32_t layer, int32_t expert, const void* x_dev, int32_t T,
                                float* y_dev, void* stream);

/*
 * Passage: the Hysen Labs page "Flash-MoE: Running a 397B Parameter Model on
 * a Laptop", section "How the SSD expert streaming pipeline works": one layer's
 * mixture-of-experts part is normalisation, routing and the shared expert
 * (second command buffer), softmax and top-K (host), then the K = 4 routed
 * experts' forward pass and their combine (third command buffer).  Here all of
 * it is one launch (batch-1) or one stream of launches (grouped path).
 * One full mixture-of-experts layer:
 *   h_out = h_in + sum_k w_k * E_{idx_k}(z) + E_shared(z)
 * with z, idx, w as in fmoe_route, accumulated in fp32 and rounded once to bf16.
 *   h_in_dev, h_out_dev : bf16 [T][H], must not overlap;
 *   idx_out_dev (int32 [T][K]) and w_out_dev (fp32 [T][K]) may be NULL.
 * T < 8 runs the fused single-token kernel once per token; T >= 8 the grouped
 * batched path when the context has one (n_experts <= 1023, max_tokens <=
 * 16320), else the single-token kernel per token (see FMOE_FLAG_*).  T == 0
 * is a no-op.  Errors: INVALID_ARG, ALIGNMENT, CUDA.
 */
FMOE_API fmoe_status fmoe_layer_forward(fmoe_ctx* ctx, int32_t layer, const void* h_in_dev, int32_t T, void* h_out_dev,
                               int32_t* idx_out_dev, float* w_out_dev, void* stream);

/*
 * Passage: the Hysen Labs page's section "How the SSD expert streaming
 * pipeline works": 60 layers each run the same per-layer sequence, and the
 * previous layer's expert command buffer is still in flight when the next
 * layer starts; the wiki page "Flash-MoE" (Performance Results) quotes the
 * resulting decode rates for the 4-bit and 2-bit expert sets.
 * Layers layer_begin .. layer_end-1 in sequence (a mixture-of-experts-only
 * stack: each layer's output is the next layer's input), equivalent to
 * chaining fmoe_layer_forward bit for bit; intermediate activations live in
 * the context workspace.  h_in_dev and h_out_dev (bf16 [T][H]) must not
 * overlap.  On the batch-1 kernel a range of two or more layers runs as one
 * launch per token through every layer (the next layer's router rows and
 * shared expert stream in while a layer finishes); FMOE_FLAG_STACK_PER_LAYER
 * makes it one launch per layer and token.  The grouped path runs layer by
 * layer.
 */
FMOE_API fmoe_status fmoe_stack_forward(fmoe_ctx* ctx, int32_t layer_begin, int32_t layer_end, const void* h_in_dev,
                               int32_t T, void* h_out_dev, void* stream);

/*
 * fmoe_layer_forward / fmoe_stack_forward on HOST buffers: h_in_host (bf16
 * [T][H]) is brought into the context's device staging buffer, the device
 * path runs on it, and h_out_host (bf16 [T][H]) and, when not NULL,
 * idx_out_host (int32 [T][K]) and w_out_host (fp32 [T][K]) receive the
 * results.  When every buffer is page-locked and mapped into the device's
 * address space (cudaHostAlloc, or cudaHostRegister with mapping; h_in_host
 * 16-byte aligned), lies inside one page-locked allocation (checked through the
 * driver's pointer range) and the call runs on the batch-1 kernel, no copy
 * engine is involved: a small kernel reads the input over the host link and the fused
 * kernel writes the outputs straight into host memory.  Otherwise (pageable
 * buffers, or the grouped path) each buffer is one cudaMemcpyAsync; pageable
 * copies block the host.  Everything is enqueued on `stream` and the call
 * returns without synchronising; the caller synchronises `stream` before
 * reading the outputs and keeps the buffers alive until then.  The input is
 * staged per context before anything is written, so h_in_host and h_out_host
 * may be the same buffer.
 * Results are bit-identical to the device-pointer calls.  Errors: as the
 * device-pointer calls (no alignment rule on host buffers), FMOE_ERR_CUDA when
 * a copy cannot be enqueued.
 */
FMOE_API fmoe_status fmoe_layer_forward_host(fmoe_ctx* ctx, int32_t layer, const void* h_in_host, int32_t T,
                                             void* h_out_host, int32_t* idx_out_host, float* w_out_host, void* stream);
FMOE_API fmoe_status fmoe_stack_forward_host(fmoe_ctx* ctx, int32_t layer_begin, int32_t layer_end,
                                             const void* h_in_host, int32_t T, void* h_out_host, void* stream);

/*
 * Writes expert `expert` (-1: shared) of `layer` back in the canonical format
 * into dst_dev (fmoe_expert_bytes bytes).  Used to check the packed layout
 * round trip.
 */
FMOE_API fmoe_status fmoe_unpack_expert(fmoe_ctx* ctx, int32_t layer, int32_t expert, void* dst_dev, void* stream);

/*
 * Synchronises `stream`, reads the device status word and clears it.
 * *device_status (may be NULL) receives the raw word (0 = no fault).  Returns
 * FMOE_ERR_TIMEOUT when a bounded wait ran out since the last poll, FMOE_OK
 * otherwise.  The context stays usable after a timeout: every launch tags its
 * cross-block results with a fresh epoch, so nothing from the failed launch is
 * read by the next one.
 */
FMOE_API fmoe_status fmoe_poll_status(fmoe_ctx* ctx, void* stream, uint32_t* device_status);

/*
 * 4-bit -> 2-bit requantisation of canonical expert blobs: the conversion of
 * the page "Flash-MoE Inference Engine", section "Weight Preparation" (step 3,
 * optional 2-bit requantisation), which names the step but not its algorithm.
 * Every 64-column group of every row of gate, up and down is refitted on its
 * own with an affine grid spanning the group's smallest and largest weight,
 * each step one IEEE fp32 operation rounded to nearest even:
 *   w = fma(q4, s4, b4); lo, hi = min, max of the group's w;
 *   s2 = bf16((hi - lo) / 3); b2 = bf16(lo); inv = s2 > 0 ? 1 / s2 : 0;
 *   q2 = min(max(rint((w - b2) * inv), 0), 3).
 *   src_dev : n_blobs contiguous canonical 4-bit blobs (fmoe_expert_bytes(H, I, 4)
 *             bytes each), device memory, read only;
 *   dst_dev : n_blobs contiguous canonical 2-bit blobs (fmoe_expert_bytes(H, I, 2)
 *             bytes each), device memory, written; must not overlap src_dev.
 * Needs no context; asynchronous on `stream` (a cudaStream_t as void*).  Both
 * pointers 16-byte aligned, H and I positive multiples of 64.  Errors
 * (INVALID_ARG, ALIGNMENT, UNSUPPORTED for H*I > 2^30, CUDA) are reported before
 * any GPU work where possible, with detail in fmoe_last_error(NULL).
 */
FMOE_API fmoe_status fmoe_requant_4to2(const void* src_dev, int32_t n_blobs, int32_t hidden, int32_t inter,
                                       void* dst_dev, void* stream);

/*
 * Timing hook for the grouped (batched) path, for benchmarks; no counterpart on
 * the pages.  While set, every call that takes the grouped path records
 * events[0] / events[1] on its stream immediately before / after the grouped
 * gate/up GEMM launch, and events[2] / events[3] around the grouped down GEMM
 * launch, so cudaEventElapsedTime gives each GEMM's device time.  `events`
 * points to 4 cudaEvent_t handles (passed as void*) owned by the caller and
 * created on the context's device; the library copies the handles and never
 * creates, synchronises or destroys them.  NULL clears the hook.  Returns
 * FMOE_ERR_INVALID_ARG for an invalid context or a NULL handle in the array.
 */
FMOE_API fmoe_status fmoe_set_gemm_events(fmoe_ctx* ctx, void* const* events);

/*
 * Phase-timing hook of the fused single-token kernel, for profiling; no
 * counterpart on the pages.  While set, a library built with FMOE_TRACE
 * (build.py --trace) records %globaltimer stamps into trace_dev, an unsigned
 * 64-bit device array [grid][fmoe_trace_layers()][fmoe_trace_points()] (grid =
 * the device's SM count; the first fmoe_trace_layers() layers of a launch),
 * owned by the caller and overwritten by every launch.  The product library
 * compiles the recording out and ignores the pointer.  NULL clears the hook.
 * Errors: INVALID_ARG (context), ALIGNMENT.
 */
FMOE_API fmoe_status fmoe_set_trace(fmoe_ctx* ctx, void* trace_dev);
FMOE_API int32_t fmoe_trace_points(void);
FMOE_API int32_t fmoe_trace_layers(void);

/*
 * Test hook: sets the context's launch epoch (the tag counter of its
 * cross-block words) on `stream` and synchronises it.  A launch tags its words
 * epoch + 1 .. epoch + layers; before those would pass 2^32 - 1 the library
 * clears the tagged words and restarts the count at 0, so setting the epoch
 * just below 2^32 exercises that wrap in a few launches.  No counterpart on the
 * pages.  Errors: INVALID_ARG (context), CUDA.
 */
FMOE_API fmoe_status fmoe_debug_set_epoch(fmoe_ctx* ctx, uint32_t epoch, void* stream);

/* Releases the workspace; the context pointer is invalid afterwards (later
 * calls with it return FMOE_ERR_INVALID_ARG).  Does not free caller memory. */
FMOE_API fmoe_status fmoe_destroy(fmoe_ctx* ctx);

/* One-line description of the last error on `ctx` (or of the last failed
 * fmoe_create when ctx is NULL).  Valid until the next call on that context. */
FMOE_API const char* fmoe_last_error(const fmoe_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* FMOE_H */
