/*
 * pw.h -- C ABI of the B200 fused mixed-precision MoE layer (PagedWeight's
 * hot path).
 *
 * What the library computes.  One Mixture-of-Experts FFN layer whose expert
 * weights are stored as Any-Precision bit-plane pages plus per-row lookup
 * tables, each linear-block (expert x projection) at its own bitwidth, with
 * routing, expert activation and the weighted output sum fused into the same
 * GPU pass:
 *   - PagedWeight (arxivlens summary), abstract paragraph: a fused
 *     mixed-precision MoE kernel processes AP bit-planes and LUTs of the
 *     GPU-resident pages; page movement runs asynchronously, overlapped with
 *     serving.
 *   - PagedWeight (legiblepapers summary), "Key Takeaways" and FAQ Q5: the
 *     kernel reads the bit-plane and LUT buffers directly, supports a
 *     different bitwidth for every linear-block, and fuses routing, expert
 *     activation and output accumulation.
 *   - same summary, "Summary & Methodology Analysis": the bit-plane and LUT
 *     buffers are GPU-resident pages that are reloaded or offloaded
 *     asynchronously to hide latency.
 *
 * Definitions (readings where the pages are silent):
 *   Linear-block W, rows x cols, applied as y = W x.  Routed expert e has
 *   block ids 3e+0 (gate, F x H), 3e+1 (up, F x H), 3e+2 (down, H x F); the
 *   shared expert (if any) has ids 3E+0..3E+2 with S in place of F.
 *   Bit-planes: plane 0 holds the MOST significant code bit; in the word
 *   covering columns 32w..32w+31 of a row, bit (i % 32) is column i; pad bits
 *   are zero.  A b-bit view reads planes 0..b-1 only:
 *   code_b = sum_{k<b} bit_k << (b-1-k) = code_{n_max} >> (n_max - b).
 *   Pages: each plane is one page.  The library reads a block's n_max planes
 *   in its paged layout: tile groups of 128 rows x 8 words, each holding the
 *   n_max planes' 4 KB tiles one after the other (so the b active planes of a
 *   group are one contiguous b * 4 KB run); rows' 16-byte halves are swapped
 *   on rows with bit 2 set (csrc/pages.h).  A block takes n_max *
 *   pw_plane_bytes(rows, cols) bytes; pw_repack_planes converts the
 *   row-major layout [plane][rows][words] into it.
 *   LUT of bitwidth b: fp16 [rows][2^b]; W[o][i] = LUT_b[o][code_b(o, i)].
 *   Router: logit[t][e] = x_t . Wr_e (+ bias_e) in fp32; experts ranked by
 *   logit, ties to the lower index; the first k are selected in that order;
 *   p = softmax over all E logits; slot weight = p of the selected expert,
 *   divided by the sum over the k selected when renorm_topk = 1.
 *   Expert: h = silu(x Wg^T) * (x Wu^T), silu(g) = g / (1 + exp(-g));
 *   y_e = h Wd^T.  Output: y_t = sum_j w_tj * y_{e_tj}(x_t) + shared(x_t)
 *   (the shared expert is added with weight 1), rounded to bf16 (nearest
 *   even); accumulation is fp32.
 *
 * Conventions.
 *   Ownership: the caller owns every buffer it passes (device buffers and
 *   pinned host copies) and keeps them alive and unmodified, except through
 *   this library, until pw_destroy.  The library owns its handle, workspace
 *   and events.
 *   Streams: pw_stream_t is a cudaStream_t (NULL = the legacy default
 *   stream).  Calls enqueue work and return without synchronising, except
 *   pw_moe_forward_host, pw_check_device_error and pw_destroy.
 *   Errors: every call returns a pw_status_t; nothing is thrown across the
 *   ABI; pw_last_error() gives a message for the calling thread.  On an
 *   error nothing has been enqueued, unless the status is PW_ERR_CUDA.
 *   Threads: a handle is used by one host thread at a time.
 *   Alignment: device buffers 16-byte aligned; x and y row-major, contiguous.
 *   Kernels: when H, F and S are multiples of 128 the expert passes run on the
 *   tensor-core kernel (TMA + tcgen05; activations are fed to it as fp16, so
 *   |x| and |silu(g) u| must stay below 65504); other shapes run on the
 *   CUDA-core kernel in fp32.  pw_linear takes the tensor-core kernel when
 *   cols is a multiple of 128.  At prefill-sized batches (routed slots
 *   averaging at least 64 tokens per expert, and max_tokens giving at least
 *   256 sorted positions: max_tokens * (top_k + (shared_ffn > 0)) >= 256)
 *   the tensor-core passes work on 256-token chunks, gate and up as separate
 *   launches with the gate output kept in a workspace buffer; the result is
 *   the same computation (PW_PREFILL=0/1 in the environment forces either).
 *   At decode both tensor-core passes run in one launch (gate/up items, then
 *   down items, each down item waiting on its expert's gate/up items).  That
 *   launch has one CTA per SM and is cooperative: the driver either makes
 *   every CTA resident at once or refuses the launch (PW_ERR_CUDA), so the
 *   waits cannot stall on a CTA that never started (for instance when MPS or
 *   another context holds SMs).
 *   Environment switches, for tests and measurements only: PW_FUSED=0 (two
 *   decode launches), PW_PREFILL=0/1, PW_DOWN_SPLIT=n (K splits of the down
 *   items), PW_FORCE_SIMPLE=1 (CUDA-core kernel; read at pw_moe_create),
 *   PW_COOP=0 (fused launch without the cooperative attribute), and for the
 *   failure-detection test PW_TEST_WAIT_US=n (device wait limit, default 2 s)
 *   with PW_TEST_STALL_GROUP=g (expert g's down items wait for a gate/up count
 *   that never arrives, so the bounded wait runs out and the forward reports
 *   PW_ERR_TIMEOUT through pw_check_device_error).
 */
#ifndef PW_H_
#define PW_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PW_ABI_VERSION 1
#define PW_MAX_BITS 8        /* n_max <= 8 */
#define PW_MAX_EXPERTS 128   /* routed experts per layer */
#define PW_MAX_TOPK 8

typedef struct pw_moe pw_moe_t; /* opaque */
typedef void* pw_stream_t;      /* cudaStream_t */

typedef enum {
  PW_OK = 0,
  PW_ERR_INVALID_ARG = 1, /* a null pointer, a size out of range, misalignment */
  PW_ERR_CUDA = 2,        /* a CUDA runtime call failed (message has the name) */
  PW_ERR_OOM = 3,         /* workspace allocation failed */
  PW_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up */
  PW_ERR_STATE = 5,       /* call not valid now (e.g. a switch still pending) */
  PW_ERR_UNSUPPORTED = 6  /* shape or device the kernels do not handle */
} pw_status_t;

typedef struct {
  int32_t hidden;      /* H, multiple of 8 */
  int32_t ffn;         /* F, routed expert FFN width, >= 1 */
  int32_t n_experts;   /* E, 1..PW_MAX_EXPERTS */
  int32_t top_k;       /* k, 1..min(E, PW_MAX_TOPK) */
  int32_t shared_ffn;  /* S, shared expert FFN width, 0 = none */
  int32_t n_max;       /* planes stored per block, 1..PW_MAX_BITS */
  int32_t renorm_topk; /* 1 = selected weights renormalised to sum to one */
  int32_t max_tokens;  /* largest T a forward may pass (sizes the workspace) */
} pw_moe_config_t;

/* One linear-block page (see "Definitions").  rows and cols follow from the
 * block id and the config. */
typedef struct {
  uint32_t* d_planes;   /* device, the block's n_max plane pages (paged
                           layout, n_max * pw_plane_bytes); planes 0..bits-1 must
                           be resident at create; the library writes planes
                           bits..n_max-1 when a switch raises the bitwidth */
  uint16_t* d_lut[2];   /* device, two LUT slots of rows * 2^n_max fp16 each;
                           slot 0 holds LUT_bits at create; the library writes
                           the idle slot when a switch changes the bitwidth */
  const uint32_t* h_planes; /* host master copy of all n_max plane pages (pinned
                               for overlap), or NULL if the block is never raised */
  const uint16_t* h_lut[PW_MAX_BITS + 1]; /* host LUT_b at index b, [rows][2^b],
                                             NULL where b is never used */
  int32_t bits;         /* bitwidth at create, 1..n_max */
} pw_block_desc_t;

/* Create a layer over caller-owned pages.  blocks has 3*E (+3 if S > 0)
 * entries in block-id order.  Allocates the workspace on the current device
 * (pw_workspace_bytes gives its size). */
pw_status_t pw_moe_create(const pw_moe_config_t* cfg, const pw_block_desc_t* blocks,
                          int32_t n_blocks, pw_moe_t** out);

/* Change the bitwidth of one linear-block (an asynchronous page move).
 * Enqueued on side_stream after the most recently issued forward ends:
 * raising b -> b' copies planes b..b'-1 and LUT_b' from the host copies;
 * lowering copies LUT_b' only (the top b' planes are already resident).  The
 * LUT lands in the idle slot, so no forward ever reads memory being written.
 * When it takes effect (PagedWeight, legiblepapers "Summary & Methodology
 * Analysis": pages move asynchronously to hide latency): every forward issued
 * afterwards checks, without blocking (cudaEventQuery), whether the copy has
 * completed; the first forward that finds it complete uses the new bitwidth.
 * A change still pending after max_lag more forwards (pw_set_switch_lag,
 * default 8) takes effect at the next forward, which then waits on the GPU
 * for the copy.  pw_get_forward_bits reports the bitwidths each forward used.
 * Forwards of one handle go on one stream (the copy is ordered after the
 * last issued forward through an event on that stream).  PW_ERR_STATE while
 * an earlier change of the same block has not taken effect yet;
 * PW_ERR_INVALID_ARG (nothing enqueued) when the host LUT for new_bits is
 * NULL, or when raising the width of a block whose host planes are NULL. */
pw_status_t pw_set_block_bits(pw_moe_t* h, int32_t block_id, int32_t new_bits,
                              pw_stream_t side_stream);

/* y = MoE(x): d_x bf16 [T][H], d_router_w fp32 [E][H], d_router_bias fp32
 * [E] or NULL, d_y bf16 [T][H] (device).  0 <= T <= max_tokens.  The
 * forward's kernels are launched with programmatic dependent launch: each
 * may be scheduled while its predecessor on the stream drains, and waits for
 * that predecessor's completion before it reads or writes anything; the
 * stream order seen by the caller is unchanged. */
pw_status_t pw_moe_forward(pw_moe_t* h, const uint16_t* d_x, int32_t T,
                           const float* d_router_w, const float* d_router_bias,
                           uint16_t* d_y, pw_stream_t stream);

/* Bytes of device workspace pw_moe_create allocates for cfg on the current
 * device (one allocation: routing lists, gathered activations, the SwiGLU
 * activations, the down pass's per-split partials -- shared with the
 * prefill gate outputs, which are dead by the time the down pass writes --
 * and the host-forward staging rows).  No allocation is made. */
pw_status_t pw_workspace_bytes(const pw_moe_config_t* cfg, int64_t* bytes);

/* Free the workspace and events after all work of the handle has finished
 * (synchronises on the handle's events).  NULL is accepted. */
pw_status_t pw_destroy(pw_moe_t* h);

/* ---- helpers beyond the four-call contract ---------------------------- */

/* pw_moe_forward with HOST activations: copies x_host (bf16 [T][H]) in and
 * y_host out through a library-owned device staging buffer, and returns
 * after the stream has finished (pinned host buffers give full copy speed). */
pw_status_t pw_moe_forward_host(pw_moe_t* h, const uint16_t* x_host, int32_t T,
                                const float* d_router_w, const float* d_router_bias,
                                uint16_t* y_host, pw_stream_t stream);

/* Bytes of one plane page of a rows x cols block (0 for a bad shape). */
int64_t pw_plane_bytes(int32_t rows, int32_t cols);

/* Convert n_planes row-major planes d_src [n_planes][rows][ceil(cols/32)]
 * into the paged layout of an n_max = n_planes block, d_dst
 * (n_planes * pw_plane_bytes bytes), on stream. */
pw_status_t pw_repack_planes(const uint32_t* d_src, uint32_t* d_dst, int32_t rows, int32_t cols,
                             int32_t n_planes, pw_stream_t stream);

/* One dequantised linear-block on its own: d_y[t][o] = sum_i W_b[o][i] x[t][i]
 * with fp32 output.  d_planes: a block of n_max planes in the paged layout
 * (bits <= n_max are read), d_lut [rows][2^bits]
 * fp16, d_x bf16 [T][cols], d_y fp32 [T][rows]; T >= 0, bits 1..8.  Uses the
 * same dequantisation and contraction as the MoE experts.  Its device waits
 * are bounded like the forward's, but it has no handle and so no device
 * error word: a wait that gives up leaves d_y unspecified without a report. */
pw_status_t pw_linear(const uint32_t* d_planes, const uint16_t* d_lut, int32_t rows,
                      int32_t cols, int32_t n_max, int32_t bits, const uint16_t* d_x,
                      int32_t T, float* d_y, pw_stream_t stream);

/* Bitwidth of a block as of the most recently issued forward (the one the
 * create call set, before any forward), and the width of a change still
 * pending (0 if none). */
pw_status_t pw_get_block_bits(const pw_moe_t* h, int32_t block_id, int32_t* bits_active,
                              int32_t* bits_pending);

/* The bitwidth every block had in the most recently issued forward (the
 * create-time widths before any forward), in block-id order; bits has room
 * for n >= 3E (+3) entries.  Lets a caller replay exactly what each forward
 * computed while page moves land asynchronously. */
pw_status_t pw_get_forward_bits(const pw_moe_t* h, int32_t* bits, int32_t n);

/* Largest number of forwards a page move may stay pending before a forward
 * waits for its copy (>= 0; 0 = the next forward always waits and uses the
 * new width). */
pw_status_t pw_set_switch_lag(pw_moe_t* h, int32_t max_lag);

/* Routing of the most recent forward: d_idx int32 [T][k] (selection order)
 * and d_w fp32 [T][k], copied device-to-device on stream. */
pw_status_t pw_get_routing(const pw_moe_t* h, int32_t* d_idx, float* d_w,
                           pw_stream_t stream);

/* Online routing statistics: the planner's "routing mass", how often each
 * expert is used (PagedWeight, legiblepapers "Summary & Methodology
 * Analysis" and FAQ Q4/Q8: damage per released byte weighs offline
 * sensitivity, online routing mass and prompt residuals).  Every forward's
 * route kernel adds, for each routed expert e, the number of (token, slot)
 * assignments to e and the sum of their routing weights (the weights the
 * combine applies), accumulated on the device in 64-bit counters and
 * doubles.  This call copies them into the host arrays counts [E] and mass
 * [E] after the forwards issued so far on stream, zeroes them if reset != 0,
 * and returns once the copies have landed (it synchronises stream). */
pw_status_t pw_routing_stats(pw_moe_t* h, uint64_t* counts, double* mass, int32_t reset,
                             pw_stream_t stream);

/* ---- residency paging --------------------------------------------------- */

/* Switch the handle to library-owned plane storage (PagedWeight,
 * legiblepapers "Summary & Methodology Analysis": the bit-plane buffers are
 * GPU-resident pages that are reloaded or offloaded asynchronously; cortexa
 * abstract: freeing weight memory for the KV cache).  Every block then holds
 * exactly its current bitwidth's planes on the device, in the paged layout
 * with that many planes per tile group, in a memory pool the library
 * creates on the handle's device.  Lowering a block's width offloads planes
 * (new storage with fewer planes replaces the old one, which is freed to
 * the pool once no issued forward can read it); raising it reloads planes
 * from the host master copy, so every block needs h_planes (else
 * PW_ERR_INVALID_ARG).  The switch semantics of pw_set_block_bits are
 * unchanged; a pool allocation that fails there is PW_ERR_OOM with nothing
 * changed.  The call copies the resident planes out of the caller's
 * d_planes on stream and returns after those copies and every forward
 * issued so far have finished: the caller may then free its plane buffers
 * (the LUT slots stay caller-owned).  PW_ERR_STATE while a bitwidth change
 * is pending.  Idempotent. */
pw_status_t pw_enable_paging(pw_moe_t* h, pw_stream_t stream);

/* Pack every block's resident planes into one new allocation of the pool
 * and free the old storage, so the memory that page moves left scattered
 * across the pool's mappings can go back to the device (pw_resident_bytes
 * with pool_reserved trims the pool).  Enqueued on stream after the last
 * issued forward; pass the stream the forwards run on (their next forward
 * then reads the packed copy).  PW_ERR_STATE without paging or while a
 * bitwidth change is pending; PW_ERR_OOM (nothing changed) if the pool
 * cannot hold a second copy of the resident planes. */
pw_status_t pw_compact_pages(pw_moe_t* h, pw_stream_t stream);

/* Device bytes of plane pages the handle keeps resident (a block's
 * resident planes x its plane page size, plus the storage of pending
 * changes; without paging, n_max planes per block).  If pool_reserved is
 * not NULL, the call first waits for the handle's issued work, returns the
 * pool's unused memory to the device (cudaMemPoolTrimTo) and reports what
 * the pool still reserves. */
pw_status_t pw_resident_bytes(pw_moe_t* h, int64_t* plane_bytes, int64_t* pool_reserved);

/* ---- the quality-aware release planner (host only) --------------------- */

/* One linear-block as the planner sees it. */
typedef struct {
  int32_t bits;          /* current bitwidth, 1..8 */
  int32_t min_bits;      /* lowest width the planner may choose, 1..bits */
  int64_t plane_bytes;   /* bytes of one plane page (pw_plane_bytes) */
  int32_t rows;          /* LUT rows (the block's output rows) */
  double mass;           /* routing mass of the block's expert (from
                            pw_routing_stats; the shared expert's is the
                            token count), >= 0 */
  double resid;          /* prompt-residual weight, >= 0 */
  double sens[PW_MAX_BITS + 1]; /* sens[b]: offline damage of the step b -> b-1 */
} pw_plan_block_t;

/* Greedy release plan (PagedWeight, legiblepapers "Summary & Methodology
 * Analysis" and FAQ Q8: the planner frees a target number of bytes by
 * picking, one at a time, the quantisation action with the least damage per
 * released byte; damage combines offline sensitivity, online routing mass
 * and prompt residuals).  Reading of the pages: an action lowers one block
 * by one bit, b -> b-1 (b > min_bits), releasing its plane page b-1 and half
 * of its LUT: plane_bytes + rows * 2^(b-1) * 2 bytes; its damage is
 * sens[b] * mass * (1 + resid), evaluated in double in that order; the
 * action with the smallest damage / bytes (double division) goes first,
 * ties to the lower block index; actions stop once the released bytes
 * reach target_bytes.  Writes the chosen width of every block to new_bits
 * [n], the bytes released and the summed damage, and *reached = 1 if the
 * target was met (0: every block ended at min_bits short of it).  Pure host
 * computation; apply the plan with pw_set_block_bits. */
pw_status_t pw_plan_release(const pw_plan_block_t* blocks, int32_t n, int64_t target_bytes,
                            int32_t* new_bits, int64_t* released, double* damage,
                            int32_t* reached);

/* Synchronises the device and reports a device-side error flag of the handle
 * (PW_ERR_TIMEOUT if a bounded wait gave up) and clears it. */
pw_status_t pw_check_device_error(pw_moe_t* h);

/* Per-launch timing for benchmarks.  While enabled, every forward records
 * CUDA events between its launch slots: route; gather + gate/up (the one
 * fused launch at decode, both prefill launches at prefill); down (empty
 * when fused); combine.
 * pw_profile_read synchronises on them and writes, for each launch slot, the
 * milliseconds summed over the forwards issued since the previous read (ms
 * has room for n >= 4 floats); *n_forwards receives how many were summed. */
pw_status_t pw_profile_enable(pw_moe_t* h, int32_t on);
pw_status_t pw_profile_read(pw_moe_t* h, float* ms, int32_t n, int32_t* n_forwards);

/* Number of kernel launches one forward of this handle issues for T tokens. */
int32_t pw_forward_launches(const pw_moe_t* h, int32_t T);

/* ---- routing without device allocation ------------------------------- */

/* The router alone, allocating nothing: the same routing as pw_moe_forward
 * (logits, top-k, softmax, per-expert bucketing in one launch), with its
 * scratch in one fixed device array of PW_ROUTE_STATIC_SCRATCH_BYTES per
 * device instead of a handle's workspace.  The PagedWeight pages have no
 * counterpart of this call; it serves callers that cannot allocate device
 * memory where they route (all of HBM already handed to weight pages and KV
 * cache, or no room for cudaMalloc's implicit device synchronisation in the
 * middle of an asynchronous page move).
 *   d_x bf16 [T][hidden], d_router_w fp32 [n_experts][hidden],
 *   d_router_bias fp32 [n_experts] or NULL (device, caller-owned);
 *   d_idx int32 [T][top_k] and d_w fp32 [T][top_k] receive the selected
 *   experts in selection order and their weights, exactly as pw_get_routing
 *   reports them after a forward of the same x.
 *   0 <= T <= PW_ROUTE_STATIC_MAX_TOKENS, 1 <= top_k <= min(n_experts, 8),
 *   n_experts <= 128, renorm_topk 0 or 1; anything else is PW_ERR_INVALID_ARG
 *   with nothing enqueued.  T = 0 returns PW_OK at once.
 * Every call made outside a stream capture looks up the array's address
 * (cudaGetSymbolAddress; PW_ERR_CUDA if that fails), so the address stays
 * right after a cudaDeviceReset, and caches it per device; a call made while
 * its stream is being captured uses the cached address, so make the first
 * call on a device before any stream capture there (PW_ERR_STATE otherwise).
 * Races: the array is shared by every call on the device in the process.  Two
 * calls whose kernels can overlap (different streams without an event between
 * them, or several host threads) corrupt each other's scratch and results;
 * the caller serialises calls per device, e.g. by issuing them all on one
 * stream. */
/* Launch geometry of the route kernel for T tokens, E experts, hidden H and
 * top_k: pure host arithmetic (no device call, so it also runs without a
 * GPU).  out[0..11] = blocks per cluster, expert groups per cluster, tokens
 * per cluster, tokens per block, experts per block, columns per staged
 * chunk, clusters, register-tile tokens, register-tile experts, selections
 * staged in shared memory for the bucketing (0/1), shared-memory offset of
 * the cluster's logits, dynamic shared memory bytes per block.
 * PW_ERR_INVALID_ARG unless 0 <= T, 1 <= E <= 128, H >= 1 and
 * 1 <= top_k <= min(E, 8). */
pw_status_t pw_route_geometry(int32_t T, int32_t E, int32_t H, int32_t top_k, int64_t* out);

#define PW_ROUTE_STATIC_MAX_TOKENS 256
#define PW_ROUTE_STATIC_SCRATCH_BYTES 25600 /* offsets, per-expert lists and a ticket */
pw_status_t pw_route_static(const uint16_t* d_x, const float* d_router_w,
                            const float* d_router_bias, int32_t T, int32_t hidden,
                            int32_t n_experts, int32_t top_k, int32_t renorm_topk,
                            int32_t* d_idx, float* d_w, pw_stream_t stream);

const char* pw_last_error(void);
int32_t pw_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PW_H_ */
