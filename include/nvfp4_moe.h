/*
 * nvfp4_moe.h - C ABI of the grouped NVFP4 MoE expert forward (sm_100a).
 *
 * The forward has four steps, one entry point each, run in this order on one
 * CUDA stream:
 *
 *   1. nvfp4_moe_route_sort    group the routed (token, expert) pairs by expert
 *   2. nvfp4_moe_gate_up_silu  act = SiLU(x Wg^T) * (x Wu^T), FP32, per sorted row
 *   3. nvfp4_moe_down          y   = act Wd^T, FP32, per sorted row
 *   4. nvfp4_moe_blend         out[t] = sum_s w[t,s] * y[pos(t,s)], token order
 *
 * plus the load-time twin builder nvfp4_moe_transpose_u8, the load-time scale
 * check nvfp4_moe_check_scales and nvfp4_moe_append_shared, which brings a
 * shared expert into the same four steps.
 *
 * Launch order.  The kernels use programmatic dependent launch: each may start
 * while the previous kernel on the stream is still running and waits for it
 * before reading what it writes.  Step 3 reads step 1's outputs before that
 * wait (to start fetching its weights early), which is safe because step 2
 * runs in between: run the four steps in this order, with no step left out,
 * on one stream (other kernels may be interleaved).
 *
 * Sources.  The operations and layouts are those of the rustdoc source pages of
 * the "metrale" project:
 *   - metrale_model_layers/layers/ops/nvfp4_moe_grouped.rs: module doc (rows
 *     grouped by expert by `moe_fp8_grouped_sort`, active experts listed,
 *     intermediates laid out by sorted position, blend
 *     `moe_weighted_sum_blend_fp8_grouped`), `Nvfp4ExpertTables`,
 *     `moe_expert_gate_up_act_nvfp4_grouped`, `moe_expert_down_act_nvfp4_grouped`;
 *   - metrale_model_arch/tp_shard/quant_shard.rs, layout comment: NVFP4 weight
 *     [N, K/2] u8 packed E2M1, weight_scale [N, K/16] u8 E4M3, one f32
 *     weight_scale_2;
 *   - metrale_model_layers/weight_map/quantized/transpose.rs,
 *     `transpose_for_gemm_gs` and its host byte loop (transpose_u8);
 *   - metrale_model_layers/weight_map/expert.rs, `ExpertWeight::null`: the MoE
 *     kernels skip a NULL expert.
 *
 * Conventions common to every entry point.
 *   - All tensor pointers are DEVICE pointers, owned by the caller, row-major
 *     and contiguous.  The library allocates no memory, never synchronises the
 *     stream and never reads device data on the host.
 *   - Return value: NVFP4_MOE_OK, or an error code from nvfp4_moe_status.
 *     Argument errors are detected on the host before any launch (nothing is
 *     launched then); a failed launch returns NVFP4_MOE_ECUDA.  Nothing is
 *     thrown across the ABI, and no kernel traps.
 *   - NVFP4 weight value:  W[n,k] = E2M1(nibble k of row n)
 *                                   * E4M3(scale[n, k/16]) * weight_scale_2.
 *     NIBBLE ORDER: byte j of a row holds k = 2j in its LOW nibble and
 *     k = 2j+1 in its HIGH nibble.  E4M3 is the finite "FN" variant (max 448);
 *     its NaN codes 0x7F / 0xFF are not valid block scales.
 *   - A pair is p = token * topk + slot.  A "sorted position" is a pair's index
 *     after grouping by expert (ascending expert id, ties by ascending p).
 *   - A NULL expert (NULL entry in its packed_ptrs table) is skipped: its rows
 *     of act / y are written as zeros.
 *   - Shape rules: hidden and intermediate are multiples of 256 (one 16-byte
 *     scale load covers 256 k); 1 <= topk <= num_experts <= 1024.
 */
#ifndef NVFP4_MOE_H_
#define NVFP4_MOE_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime.h>

#if defined(NVFP4_MOE_BUILD) && defined(__GNUC__)
#define NVFP4_MOE_API __attribute__((visibility("default")))
#else
#define NVFP4_MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_MOE_OK = 0,
  NVFP4_MOE_EINVAL = 1, /* NULL pointer or invalid argument value            */
  NVFP4_MOE_ESHAPE = 2, /* shape outside the supported set (see above)       */
  NVFP4_MOE_ECUDA = 3   /* a CUDA call or kernel launch failed               */
} nvfp4_moe_status;

/*
 * One NVFP4 projection across the routed experts (Nvfp4ExpertTables in
 * nvfp4_moe_grouped.rs).  All three are DEVICE arrays of length num_experts:
 *   packed_ptrs[e]  device pointer to expert e's packed E2M1 bytes  u8 [N, K/2]
 *                   (16-byte aligned), or NULL for a NULL expert;
 *   scale_ptrs[e]   device pointer to its E4M3 block scales          u8 [N, K/16]
 *                   (16-byte aligned);
 *   scale2[e]       its f32 weight_scale_2.
 */
typedef struct {
  const void* const* packed_ptrs;
  const void* const* scale_ptrs;
  const float* scale2;
} nvfp4_expert_tables;

/*
 * Launch options of the two projection steps (nvfp4_moe_*_ex).  A NULL pointer,
 * or a zero field, means "choose from the shape":
 *   path     0 auto; 1 decode path (register-fed warp MMA over streamed weights,
 *            for few rows per expert); 2 prefill path (tcgen05 MMA with TMEM
 *            accumulators over shared-memory-dequantised weight tiles).
 *   split    decode path: warps of a CTA that split K, 1, 2 or 4 (2 and 4
 *            with tiles = 1 and depth = 2).
 *   tiles    decode path: 8-row token tiles per pass over an expert, 1, 2 or 4
 *            (gate+up) / 1 or 2 (down); 4 takes depth = 2.
 *   depth    decode path: weight chunks each warp keeps in flight, 2 or 3.
 *   staging  decode path: how a pass holds its token rows in shared memory.
 *            1: every 256-wide K chunk is converted up front, then the
 *            weights stream with no CTA-wide step (needs K/256 x 4 KB per
 *            8-row tile, twice that for down, within 200 KB); 2: a two-chunk
 *            ring refilled chunk by chunk.  Automatic: 1 when it fits in 72 KB.
 * Every choice computes the same function; it affects speed and the FP32
 * summation order only.  A choice the shapes do not allow returns
 * NVFP4_MOE_EINVAL.
 */
typedef struct {
  int32_t path;
  int32_t split;
  int32_t tiles;
  int32_t depth;
  int32_t staging;
} nvfp4_moe_launch_opts;

/*
 * Step 1: group the routed pairs by expert (moe_fp8_grouped_sort, named in the
 * module doc of nvfp4_moe_grouped.rs).
 *
 *   topk_ids        i32 [num_tokens, topk]  expert id of each pair
 *   expert_offsets  i32 [num_experts + 1]   out: exclusive prefix of per-expert
 *                                           pair counts; [E] = kept pairs
 *   sorted_pair_ids i32 [P]                 out: pair id at each sorted position;
 *                                           positions >= kept pairs hold -1
 *   pair_pos        i32 [P]                 out: sorted position of each pair
 *                                           (inverse of sorted_pair_ids), -1 if dropped
 *   active_experts  i32 [num_experts]       out: experts with >= 1 pair, ascending,
 *                                           padded with -1
 *   active_count    i32 [1]                 out: number of active experts
 *   status          i32 [1] or NULL         out: 0, or 1 if some id was outside
 *                                           [0, num_experts) (that pair is dropped)
 * P = num_tokens * topk, at most 1<<24.  The result is unique (bit-exact).
 */
NVFP4_MOE_API int nvfp4_moe_route_sort(const int32_t* topk_ids, uint32_t num_tokens, uint32_t topk,
                         uint32_t num_experts, int32_t* expert_offsets,
                         int32_t* sorted_pair_ids, int32_t* pair_pos,
                         int32_t* active_experts, int32_t* active_count,
                         int32_t* status, cudaStream_t stream);

/*
 * Step 2: grouped gate+up with the SiLU product kept in FP32
 * (moe_expert_gate_up_act_nvfp4_grouped in nvfp4_moe_grouped.rs).
 *
 *   x           bf16 bits [num_tokens, k_hidden]
 *   gate, up    tables of [n_inter, k_hidden] NVFP4 weights
 *   act         f32 [P, n_inter]  out: row r = sorted position r:
 *               act[r, n] = SiLU(g) * u, g = sum_k Wg[n,k] x[t,k], u likewise,
 *               t = sorted_pair_ids[r] / topk.  Rows >= kept pairs are untouched.
 *   expert_offsets, sorted_pair_ids, active_experts, active_count: from step 1.
 *   cap         upper bound on active experts used to size the launch; pass
 *               nvfp4_moe_active_cap(num_experts, P).
 * Gate and up are not rounded to BF16 before SiLU.  n_inter % 64 == 0.
 */
NVFP4_MOE_API int nvfp4_moe_gate_up_silu(const uint16_t* x, nvfp4_expert_tables gate,
                           nvfp4_expert_tables up, float* act,
                           const int32_t* expert_offsets, const int32_t* sorted_pair_ids,
                           const int32_t* active_experts, const int32_t* active_count,
                           uint32_t n_inter, uint32_t k_hidden, uint32_t cap,
                           uint32_t num_tokens, uint32_t topk, cudaStream_t stream);

/* nvfp4_moe_gate_up_silu with explicit launch options (NULL = automatic). */
NVFP4_MOE_API int nvfp4_moe_gate_up_silu_ex(const uint16_t* x, nvfp4_expert_tables gate,
                              nvfp4_expert_tables up, float* act,
                              const int32_t* expert_offsets, const int32_t* sorted_pair_ids,
                              const int32_t* active_experts, const int32_t* active_count,
                              uint32_t n_inter, uint32_t k_hidden, uint32_t cap,
                              uint32_t num_tokens, uint32_t topk,
                              const nvfp4_moe_launch_opts* opts, cudaStream_t stream);

/*
 * Step 3: grouped down projection over the FP32 SiLU products
 * (moe_expert_down_act_nvfp4_grouped in nvfp4_moe_grouped.rs).
 *
 *   act     f32 [P, k_inter]   from step 2 (rows are sorted positions)
 *   down    table of [n_hidden, k_inter] NVFP4 weights
 *   y       f32 [P, n_hidden]  out: y[r, j] = sum_i Wd[j,i] act[r,i].
 *           Rows >= kept pairs are untouched.
 *   cap, num_tokens, topk: as for step 2 (P = num_tokens * topk).
 * n_hidden % 128 == 0.
 */
NVFP4_MOE_API int nvfp4_moe_down(const float* act, nvfp4_expert_tables down, float* y,
                   const int32_t* expert_offsets, const int32_t* active_experts,
                   const int32_t* active_count, uint32_t n_hidden, uint32_t k_inter,
                   uint32_t cap, uint32_t num_tokens, uint32_t topk, cudaStream_t stream);

/* nvfp4_moe_down with explicit launch options (NULL = automatic). */
NVFP4_MOE_API int nvfp4_moe_down_ex(const float* act, nvfp4_expert_tables down, float* y,
                      const int32_t* expert_offsets, const int32_t* active_experts,
                      const int32_t* active_count, uint32_t n_hidden, uint32_t k_inter,
                      uint32_t cap, uint32_t num_tokens, uint32_t topk,
                      const nvfp4_moe_launch_opts* opts, cudaStream_t stream);

/*
 * Bytes of caller-owned device workspace the tcgen05 path needs for one call
 * of nvfp4_moe_gate_up_silu_ws / nvfp4_moe_down_ws with these sizes (the two
 * steps use disjoint parts of it, so one buffer serves both).
 */
NVFP4_MOE_API size_t nvfp4_moe_workspace_bytes(uint32_t num_tokens, uint32_t topk, uint32_t hidden,
                                               uint32_t inter);

/*
 * Steps 2 and 3 with a workspace, which opens the tcgen05 path (path 2, or
 * path 0 when the output width is a multiple of 128 for gate+up, 256 for
 * down, and there are at least 2 routed rows per expert on average; path 2
 * with another width returns NVFP4_MOE_ESHAPE): activations are packed
 * once into f16 rows by sorted position (x gathered from its token; act as an
 * f16 hi + lo pair; each row scaled by a power of two into the f16 range),
 * per-expert TMA tensor maps of the weights are built on the device from the
 * tables, and the projection kernel loads weight and activation tiles with
 * TMA, decodes the weights into tensor memory (or, at 256-row passes, shared
 * memory) and runs tcgen05.mma with FP32 accumulators in tensor memory.
 * Arguments as for the calls without _ws, plus num_experts (the length of the
 * expert tables; it bounds the offsets read) and `workspace`: device memory of
 * at least nvfp4_moe_workspace_bytes(num_tokens, topk, hidden, inter) bytes,
 * 256-byte aligned (NVFP4_MOE_EINVAL otherwise), owned by the caller,
 * overwritten by the call.  For the tcgen05 path opts->tiles selects the
 * token rows per pass: 2 -> 16 and 16 -> 128 (one CTA per 128 or 256 output
 * rows); 4 -> 32, 24 -> 192 and 32 -> 256 (a cluster of two CTAs sharing each
 * MMA; down takes 192 for 32); 0 = from the shape.  Results equal the other
 * path's within FP32 rounding.  Calls on one stream may share the workspace;
 * concurrent calls may not.
 */
NVFP4_MOE_API int nvfp4_moe_gate_up_silu_ws(
    const uint16_t* x, nvfp4_expert_tables gate, nvfp4_expert_tables up, float* act,
    const int32_t* expert_offsets, const int32_t* sorted_pair_ids, const int32_t* active_experts,
    const int32_t* active_count, uint32_t n_inter, uint32_t k_hidden, uint32_t cap,
    uint32_t num_tokens, uint32_t topk, uint32_t num_experts, const nvfp4_moe_launch_opts* opts,
    void* workspace, size_t workspace_bytes, cudaStream_t stream);

NVFP4_MOE_API int nvfp4_moe_down_ws(
    const float* act, nvfp4_expert_tables down, float* y, const int32_t* expert_offsets,
    const int32_t* active_experts, const int32_t* active_count, uint32_t n_hidden, uint32_t k_inter,
    uint32_t cap, uint32_t num_tokens, uint32_t topk, uint32_t num_experts,
    const nvfp4_moe_launch_opts* opts, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Allocation-free gate+up (tcgen05 path).  The pages have no counterpart to
 * this call; it exists for callers that cannot hand the library a workspace:
 * code whose device memory is owned by another allocator or a fixed budget,
 * and code that must not call cudaMalloc, which can block on the whole device
 * or fail midway.
 *
 * Same arguments and result as nvfp4_moe_gate_up_silu_ws with path 2 and no
 * workspace.  The packed token rows go to a fixed scratch array inside the
 * library: 8 MiB of device memory on every GPU that loads the library, held
 * until the process exits.  Requests needing more than that (P * k_hidden * 2
 * bytes of rows, plus two arrays of P * 4 bytes for the row and token scale
 * exponents, each rounded up to 256, plus 512 KiB of tensor maps, P =
 * num_tokens * topk) return NVFP4_MOE_ESHAPE before anything is launched; so
 * do widths the tcgen05 path does not take (n_inter % 128, k_hidden % 256).
 * The call never allocates memory.  Its first call on a device looks the
 * scratch array's device address up (cudaGetSymbolAddress) with that device
 * current; make that first call before any stream capture.  The address is
 * kept for the life of the process: after cudaDeviceReset of a device, do not
 * call this entry point on that device again.  All calls share the one array
 * and each call leaves its packed rows there: calls whose kernels overlap on
 * the GPU (different streams, or different host threads) race on it.
 */
NVFP4_MOE_API int nvfp4_moe_gate_up_silu_noalloc(
    const uint16_t* x, nvfp4_expert_tables gate, nvfp4_expert_tables up, float* act,
    const int32_t* expert_offsets, const int32_t* sorted_pair_ids, const int32_t* active_experts,
    const int32_t* active_count, uint32_t n_inter, uint32_t k_hidden, uint32_t cap,
    uint32_t num_tokens, uint32_t topk, uint32_t num_experts, cudaStream_t stream);

/*
 * Activation of a non-gated expert (nvfp4_moe_up_act).
 */
typedef enum {
  NVFP4_MOE_ACT_RELU2 = 1, /* f(z) = max(z, 0)^2 (squared ReLU) */
  NVFP4_MOE_ACT_SILU = 2   /* f(z) = z / (1 + exp(-z))          */
} nvfp4_moe_activation;

/*
 * Step 2 for non-gated experts, which hold only an up and a down projection
 * (the routed experts whose prefill twins `prepare_prefill_weights` in
 * nemotron_moe/prefill_weights.rs builds from up and down alone).  The pages
 * do not name the activation; the caller picks it (nvfp4_moe_activation).
 *
 *   x           bf16 bits [num_tokens, k_hidden]
 *   up          table of [n_inter, k_hidden] NVFP4 weights
 *   act         f32 [P, n_inter]  out: row r = sorted position r:
 *               act[r, n] = f(sum_k Wu[n,k] x[t,k]), t = sorted_pair_ids[r] / topk.
 *               Rows >= kept pairs are untouched; a NULL expert's rows are zero.
 *   activation  NVFP4_MOE_ACT_RELU2 or NVFP4_MOE_ACT_SILU (else NVFP4_MOE_EINVAL).
 *   the rest    as for nvfp4_moe_gate_up_silu_ex.
 * n_inter % 128 == 0.  Step 3 (nvfp4_moe_down) then reads act unchanged.
 */
NVFP4_MOE_API int nvfp4_moe_up_act(const uint16_t* x, nvfp4_expert_tables up, float* act,
                                   const int32_t* expert_offsets, const int32_t* sorted_pair_ids,
                                   const int32_t* active_experts, const int32_t* active_count,
                                   uint32_t n_inter, uint32_t k_hidden, uint32_t cap,
                                   uint32_t num_tokens, uint32_t topk, int activation,
                                   const nvfp4_moe_launch_opts* opts, cudaStream_t stream);

/*
 * nvfp4_moe_up_act with a workspace, opening the tcgen05 path under the rules
 * of nvfp4_moe_gate_up_silu_ws, with an output width that is a multiple of
 * 256 (two halves of 128 rows of the one matrix per CTA).  The workspace is
 * sized by nvfp4_moe_workspace_bytes as for the gated layer.
 */
NVFP4_MOE_API int nvfp4_moe_up_act_ws(const uint16_t* x, nvfp4_expert_tables up, float* act,
                                      const int32_t* expert_offsets, const int32_t* sorted_pair_ids,
                                      const int32_t* active_experts, const int32_t* active_count,
                                      uint32_t n_inter, uint32_t k_hidden, uint32_t cap,
                                      uint32_t num_tokens, uint32_t topk, uint32_t num_experts,
                                      int activation, const nvfp4_moe_launch_opts* opts,
                                      void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Device error word of the library: 0, or 1 if a tcgen05-path kernel gave up
 * waiting on one of its barriers (its outputs are then not valid).  Kernels
 * never trap; they set this word and exit.  Reading it synchronises the
 * device; clear != 0 resets it to 0.  Returns -1 if the read itself failed.
 */
NVFP4_MOE_API int nvfp4_moe_device_error(int clear);

/*
 * Self-test of the bounded waits behind nvfp4_moe_device_error (the pages have
 * no counterpart; the device "bad" word that `nvfp4_tc_lean_repack` in
 * nvfp4_moe_grouped.rs sets for the host to read is the same pattern).  One
 * thread initialises a barrier that expects one arrival, arrives on it only if
 * `arrive` is non-zero, then waits on it with the library's bounded wait,
 * giving up after `cycle_limit` SM clock cycles.  With arrive == 0 the wait
 * runs out, the device error word becomes 1 and the kernel returns normally
 * (nothing traps; the context stays usable); with arrive != 0 the word is left
 * as it was.  cycle_limit == 0 returns NVFP4_MOE_EINVAL.  Asynchronous: read
 * the result with nvfp4_moe_device_error.
 */
NVFP4_MOE_API int nvfp4_moe_wait_selftest(uint32_t cycle_limit, int arrive, cudaStream_t stream);

/*
 * Step 4: router-weighted blend back into token order
 * (moe_weighted_sum_blend_fp8_grouped, named in the module doc of
 * nvfp4_moe_grouped.rs).
 *
 *   y            f32 [P, hidden]            from step 3
 *   topk_weights f32 [num_tokens, topk]
 *   pair_pos     i32 [P]                    from step 1 (-1 = dropped pair)
 *   out_f32      f32 [num_tokens, hidden]   out: sum over s = 0..topk-1, in that
 *                                           order, of w[t,s] * y[pair_pos[t*topk+s]]
 *   out_bf16     bf16 bits [num_tokens, hidden] or NULL: out_f32 rounded to
 *                nearest even.
 * hidden % 4 == 0.  Deterministic: no atomics.
 */
NVFP4_MOE_API int nvfp4_moe_blend(const float* y, const float* topk_weights, const int32_t* pair_pos,
                    float* out_f32, uint16_t* out_bf16, uint32_t num_tokens, uint32_t topk,
                    uint32_t hidden, cudaStream_t stream);

/*
 * The four steps of one layer in one call: nvfp4_moe_route_sort,
 * nvfp4_moe_gate_up_silu(_ws), nvfp4_moe_down(_ws) and nvfp4_moe_blend, launched
 * in that order on `stream` with cap = nvfp4_moe_active_cap(num_experts, P).
 * The results are those of the four calls (bit for bit); one call saves the
 * host three trips through the ABI.  Buffers (all DEVICE, caller-owned):
 *
 *   expert_offsets i32 [num_experts + 1]    sorted_pair_ids i32 [P]
 *   pair_pos       i32 [P]                  active_experts  i32 [num_experts]
 *   active_count   i32 [1]                  status          i32 [1] or NULL
 *   act            f32 [P, inter]           y               f32 [P, hidden]
 *   out_f32        f32 [num_tokens, hidden] out_bf16        bf16 bits [num_tokens, hidden] or NULL
 *
 * workspace / workspace_bytes as for the _ws calls, or NULL / 0 for the decode
 * path only.  Returns the first non-zero status of the four steps (the later
 * steps are then not launched).
 */
typedef struct {
  int32_t* expert_offsets;
  int32_t* sorted_pair_ids;
  int32_t* pair_pos;
  int32_t* active_experts;
  int32_t* active_count;
  int32_t* status;
  float* act;
  float* y;
  float* out_f32;
  uint16_t* out_bf16;
} nvfp4_moe_buffers;

NVFP4_MOE_API int nvfp4_moe_forward(const uint16_t* x, const int32_t* topk_ids,
                                    const float* topk_weights, nvfp4_expert_tables gate,
                                    nvfp4_expert_tables up, nvfp4_expert_tables down,
                                    const nvfp4_moe_buffers* buffers, uint32_t num_tokens,
                                    uint32_t topk, uint32_t num_experts, uint32_t hidden,
                                    uint32_t inter, const nvfp4_moe_launch_opts* opts,
                                    void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * The four steps of one layer of non-gated experts in one call:
 * nvfp4_moe_route_sort, nvfp4_moe_up_act(_ws) with `activation`,
 * nvfp4_moe_down(_ws) and nvfp4_moe_blend.  Buffers, workspace and errors as
 * for nvfp4_moe_forward.
 */
NVFP4_MOE_API int nvfp4_moe_forward_nongated(
    const uint16_t* x, const int32_t* topk_ids, const float* topk_weights, nvfp4_expert_tables up,
    nvfp4_expert_tables down, const nvfp4_moe_buffers* buffers, uint32_t num_tokens, uint32_t topk,
    uint32_t num_experts, uint32_t hidden, uint32_t inter, int activation,
    const nvfp4_moe_launch_opts* opts, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Load-time twin builder: byte transpose [rows, cols] -> [cols, rows]
 * (transpose_u8, used by transpose_for_gemm_gs in transpose.rs, whose host
 * fallback loop t[j*rows + i] = b[i*cols + j] defines it).  src and dst must
 * not overlap.  Bit-exact.
 */
NVFP4_MOE_API int nvfp4_moe_transpose_u8(const uint8_t* src, uint8_t* dst, uint32_t rows, uint32_t cols,
                           cudaStream_t stream);

/*
 * Shared expert.  The launcher docs of nvfp4_moe_grouped.rs
 * (moe_expert_gate_up_act_nvfp4_grouped, moe_expert_down_act_nvfp4_grouped)
 * run a shared expert in the same gate+up and down launches as the routed
 * experts: one row per token, its own weights, outputs laid out by token.
 * Here it enters the forward as one more routing slot per token:
 *
 *   ids_out     i32 [num_tokens, topk + 1]  out: slots 0..topk-1 = topk_ids;
 *               slot topk = num_experts + t / shared_rows
 *   weights_out f32 [num_tokens, topk + 1]  out: slots 0..topk-1 = topk_weights;
 *               slot topk = shared_weights[t], or 1 when shared_weights is NULL
 *   shared_weights f32 [num_tokens] or NULL
 *
 * The caller's three tables have num_experts + S entries, S =
 * nvfp4_moe_shared_slots(num_tokens, shared_rows), entries num_experts ..
 * num_experts + S - 1 all holding the shared expert's weights (same shapes
 * as a routed expert).  Run the forward on ids_out / weights_out with topk + 1
 * slots and num_experts + S experts: out then adds shared_weights[t] times
 * the shared expert's output, and because the shared entries sort after
 * every routed expert, in token order, rows expert_offsets[num_experts] ..
 * + num_tokens - 1 of act and y are the shared expert's SiLU product and down
 * output for tokens 0 .. num_tokens - 1 (sh_act and sh_down_out).  Each block
 * of shared_rows tokens gets its own CTAs in the projections; a block size
 * near the routed rows per expert keeps the work even.
 * ESHAPE if topk or num_experts is 0, num_experts + S > 1024 or
 * num_tokens * (topk + 1) > 1<<24; EINVAL for shared_rows == 0 or a NULL
 * required pointer.  num_tokens == 0 launches nothing.
 */
NVFP4_MOE_API int nvfp4_moe_append_shared(const int32_t* topk_ids, const float* topk_weights,
                                          const float* shared_weights, uint32_t num_tokens,
                                          uint32_t topk, uint32_t num_experts,
                                          uint32_t shared_rows, int32_t* ids_out,
                                          float* weights_out, cudaStream_t stream);

/* Host helper: table entries the shared expert takes, ceil(num_tokens / shared_rows)
 * (0 for shared_rows == 0). */
NVFP4_MOE_API uint32_t nvfp4_moe_shared_slots(uint32_t num_tokens, uint32_t shared_rows);

/*
 * Load-time check of one projection's E4M3 block scales
 * (nvfp4_tc_lean_repack in nvfp4_moe_grouped.rs flags a negative or NaN
 * scale, after which the matrix is unusable).  For each expert e of the table
 * with non-NULL packed_ptrs[e] and scale_ptrs[e], ADDS to bad[e] the number of
 * its n * k / 16 scale codes that are NaN (0x7F, 0xFF) or negative (0x81 ..
 * 0xFE; 0x80 is -0 and passes).  bad: u32 [num_experts], device, zeroed by
 * the caller before the first check it collects.  scale2 is not read.
 * k % 256 == 0 (every scale row is whole 16-byte vectors), 1 <= num_experts
 * <= 1024, n * k / 16 < 2^32.  Bit-exact; the order of the adds does not
 * change the counts.
 */
NVFP4_MOE_API int nvfp4_moe_check_scales(nvfp4_expert_tables t, uint32_t num_experts, uint32_t n,
                                         uint32_t k, uint32_t* bad, cudaStream_t stream);

/*
 * Tensor-parallel shard of NVFP4 weights at load time (shard_quantized_nvfp4 in
 * metrale_model_arch/tp_shard/quant_shard.rs).  A stack of num_matrices
 * matrices [n, k]: packed u8 [num_matrices, n, k/2], scale u8
 * [num_matrices, n, k/16], back to back.  Writes this rank's part of each into
 * packed_out / scale_out, stacked the same way:
 *   NVFP4_MOE_SHARD_COLUMN  rows rank*n/tp .. (rank+1)*n/tp - 1 of both tensors
 *                           (gate / up: each rank holds n/tp intermediate rows);
 *                           out [num_matrices, n/tp, k/2] and [.., n/tp, k/16]
 *   NVFP4_MOE_SHARD_ROW     in every row, bytes rank*k/2/tp .. of packed and
 *                           rank*k/16/tp .. of scale (down: each rank holds k/tp
 *                           of the intermediate); out [.., n, k/2/tp], [.., n, k/16/tp]
 * weight_scale_2 is per tensor and the same on every rank (not touched here).
 * tp = 1 copies the whole stack.  A rank's partial outputs of the forward then
 * sum over ranks to the unsharded result (one all-reduce of out).
 * ESHAPE: k % 16, n % tp (column), k % tp, (k/2) % tp or (k/16) % tp (row).
 * EINVAL: bad kind, tp == 0, rank >= tp, NULL or overlapping buffers.
 * The forward's own shape rules (multiples of 256 for k, 64 / 128 for n)
 * apply to the shards.  Bit-exact.
 */
typedef enum { NVFP4_MOE_SHARD_COLUMN = 0, NVFP4_MOE_SHARD_ROW = 1 } nvfp4_moe_shard_kind;

NVFP4_MOE_API int nvfp4_moe_shard_nvfp4(const uint8_t* packed, const uint8_t* scale,
                                        uint32_t num_matrices, uint32_t n, uint32_t k, int kind,
                                        uint32_t rank, uint32_t tp, uint8_t* packed_out,
                                        uint8_t* scale_out, cudaStream_t stream);

/*
 * Load-time concatenated / padded twins (transpose_concat_for_gemm_gs and
 * transpose_concat_for_gemm_padded in transpose.rs, whose host loops define
 * the result).  num_parts weights share K; part p is packed u8 [n_p, k/2] and
 * scale u8 [n_p, k/group_size] (group_size 16 for NVFP4, 32 for MXFP4).
 * packed_parts, scale_parts and part_rows are HOST arrays of length num_parts
 * (the first two hold device pointers).  Writes
 *   packed_out u8 [k/2, stride]          column n_off + i of row j = part p's
 *   scale_out  u8 [k/group_size, stride] byte (i, j), n_off = rows of parts < p;
 * columns sum(n_p) .. stride - 1 are zero.  stride = sum(n_p) is the plain
 * concatenation; one part with stride = n_0 is transpose_for_gemm_gs.  Outputs
 * must not overlap the inputs or each other.  Bit-exact.
 * EINVAL: num_parts == 0 (the page rejects empty parts), NULL pointers.
 * ESHAPE: k odd, group_size == 0 or not dividing k, stride < sum(n_p),
 * n_p > 2097120.
 */
NVFP4_MOE_API int nvfp4_moe_transpose_concat(const uint8_t* const* packed_parts,
                                             const uint8_t* const* scale_parts,
                                             const uint32_t* part_rows, uint32_t num_parts,
                                             uint32_t k, uint32_t group_size, uint32_t stride,
                                             uint8_t* packed_out, uint8_t* scale_out,
                                             cudaStream_t stream);

/* Host helper: launch bound on active experts, min(num_experts, num_pairs). */
NVFP4_MOE_API uint32_t nvfp4_moe_active_cap(uint32_t num_experts, uint32_t num_pairs);

/* Static, human-readable name of a status code. */
NVFP4_MOE_API const char* nvfp4_moe_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_MOE_H_ */
