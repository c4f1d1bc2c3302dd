/*
 * la2.h -- C ABI of the Lightning Attention-2 library (libla2.so), sm_100a.
 *
 * The operation (per batch b and head h, identity feature map, no normaliser,
 * no 1/sqrt(d) scale inside the call):
 *
 *     o_t = sum_{s<=t} lambda_h^(t-s) (q_t . k_s) v_s
 *
 * Causal linear attention is defined on the "Lightning Attention" explainer
 * page (lizeman.github.io llm-arch-kb), section 1 "Premise" (numerator of the
 * out_t formula and the prefix-sum recurrence S_t = S_{t-1} + phi(k_t) v_t^T),
 * with phi the identity as in its section 2.  lambda_h in (0,1] is a per-head
 * decay on the lag t-s; lambda_h = 1 is the plain prefix sum.  The tiled
 * computation (intra-tile masked left product, inter-tile right product with
 * the running d x e state, state update) is the derivation of section 2,
 * steps 1-4, with the decay folded into each step; the backward uses the same
 * tiling, as the Lightning Attention-2 abstract (mlsanity.com/paper/2401.04658)
 * says, run in the reverse direction for dk and dv.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains them past the call.
 *   - q, k, dq, dk are [B, H, T, d] contiguous (d fastest); v, out, dout, dv
 *     are [B, H, T, e] contiguous.  The inputs q, k, v, dout have the element
 *     type `dtype`; the outputs out, dq, dk, dv are fp32, or, through the
 *     `_ex` / la2_bwd_state calls' out_dtype, bf16 (see la2_dtype).  Every
 *     tensor pointer must be 16-byte aligned.
 *   - decay is a device array of H floats (fp32) holding lambda_h in (0, 1];
 *     values outside that range are the caller's error and are not checked.
 *   - block is the tile length T_B (64, 128 or 256): the state is carried
 *     across blocks of that many positions, the products inside a block are
 *     the masked left product.  It changes the order of floating-point
 *     operations only, never the mathematical result.  T need not be a
 *     multiple of block: the last tile is short.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream).  Argument
 *     errors are reported synchronously and launch nothing.  A failed launch
 *     returns LA2_ERR_CUDA.  Faults detected inside a kernel (a bounded wait
 *     that ran out) are recorded in a device status word that
 *     la2_device_status() reads.
 *   - B, H or T equal to 0 is an empty problem: LA2_OK, nothing is launched
 *     and no pointer is dereferenced (except that la2_fwd_state with T = 0
 *     still sets final_state, by a device copy or memset on `stream`).
 */
#ifndef LA2_H_
#define LA2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle (a cudaStream_t / CUstream). */
typedef struct CUstream_st *la2_stream_t;

typedef enum {
    LA2_OK = 0,
    LA2_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad block/dtype, misaligned pointer */
    LA2_ERR_UNSUPPORTED = 2,  /* well-formed but not implemented for this dtype/shape; never a fallback */
    LA2_ERR_WORKSPACE = 3,    /* workspace missing or smaller than la2_workspace_bytes() */
    LA2_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed (launch, tensor-map encode, ...) */
    LA2_ERR_TIMEOUT = 5       /* a kernel's bounded wait ran out (see la2_device_status) */
} la2_status;

/*
 * Element type of the inputs (`dtype`) and of the outputs (`out_dtype`, in
 * la2_fwd_ex, la2_bwd_ex and la2_bwd_state; fp32 in every other call).
 *
 * With fp32 outputs the accuracy contract is max|out - exact| <= 2e-2 *
 * rms(exact) for bf16 inputs (1e-5 for fp32 inputs).  The outputs of this
 * operation have max/rms ~ 10, so a bf16 result's own rounding (up to 2^-8 of
 * the value, i.e. up to ~2^-5 of rms) does not fit inside that bound; with
 * out_dtype = BF16 each fp32 result is rounded to nearest even once, in the
 * kernel's output epilogue, and the contract is
 *     |out - exact| <= 2e-2 * rms(exact) + 2^-8 * |exact|   element by element.
 * BF16 outputs need BF16 inputs (fp32 inputs with BF16 outputs:
 * LA2_ERR_UNSUPPORTED); they halve the bytes the kernels write.
 */
typedef enum {
    LA2_DTYPE_F32 = 0,   /* fp32 inputs; fp32 arithmetic on SIMT cores */
    LA2_DTYPE_BF16 = 1   /* bf16 inputs; tcgen05 tensor cores, fp32 accumulation and state */
} la2_dtype;

/*
 * Memory layout of the [.., T, ..] tensors (q, k, v, out, dout, dq, dk, dv):
 * LA2_LAYOUT_BHTD is [B, H, T, D] (each sequence contiguous, the layout of the
 * "Lightning Attention" explainer's section 3 sketch, and of every entry point
 * without a layout argument); LA2_LAYOUT_BTHD is [B, T, H, D], the layout a
 * model's projections produce (positions of one sequence H*D elements apart).
 * States (init_state, final_state, decode state) are [B, H, d, e] in both.
 */
typedef enum {
    LA2_LAYOUT_BHTD = 0,
    LA2_LAYOUT_BTHD = 1
} la2_layout;

/*
 * Bytes of device workspace la2_fwd (is_bwd = 0) or la2_bwd (is_bwd = 1) needs
 * for these sizes.  The state carried along a sequence (d x e) stays on chip;
 * the workspace only holds the fp32 end state of each segment that a sequence
 * is cut into so that the work fills the GPU's 148 SMs (see la2_schedule): at
 * most 147 states of d x e floats per group of roles with the same (d, e).
 * The value does not depend on T (under AUTO it covers the plan AUTO takes at
 * any T); it depends on the schedule setting in force (la2_set_schedule).  0 means the call accepts workspace = NULL.  Returns
 * (size_t)-1 for arguments the call would reject.
 */
size_t la2_workspace_bytes(int B, int H, int T, int d, int e, int block,
                           la2_dtype dtype, int is_bwd);

/*
 * How the bf16 kernels spread the (sequence, role) units of a call over CTAs,
 * one CTA per SM (the scan of each unit is sequential in T):
 *   UNIFORM  each unit is cut into equal segments, one CTA each, when there
 *            are fewer units than SMs (otherwise one CTA per unit, in waves);
 *   BALANCED the units' 128-position tiles are laid end to end and cut into
 *            148 equal runs, one CTA each, which processes the pieces of
 *            units its run covers one after the other (one wave, equal work);
 *   AUTO     (default) the library's choice: BALANCED for at least 148
 *            units of at least 128 tiles whose UNIFORM waves would leave over
 *            a quarter of their SM time idle (e.g. 192 units: a second wave
 *            of 44 CTAs), UNIFORM elsewhere.  Measured on a B200 with the
 *            benchmark: BALANCED +5% at T = 65,536 with 64 sequences, -1% to
 *            -2% where UNIFORM cuts few units into segments or runs one
 *            partial wave, and up to 23% slower per pass where UNIFORM fills
 *            its waves (every SM busy makes each tile slower, and the
 *            pre-pass re-reads inputs).
 * A segment that starts inside its unit receives its incoming state from a
 * pre-pass over the unit's earlier positions.  Results agree between the
 * schedules to rounding (the sum is grouped differently).  Process-wide;
 * returns the previous setting, or leaves it and returns it for an unknown
 * value.  Change it only between calls; la2_workspace_bytes follows it.
 */
typedef enum {
    LA2_SCHEDULE_AUTO = 0,
    LA2_SCHEDULE_UNIFORM = 1,
    LA2_SCHEDULE_BALANCED = 2
} la2_schedule;

la2_schedule la2_set_schedule(la2_schedule schedule);

/*
 * The launch plan a bf16 la2_fwd (is_bwd = 0) or la2_bwd (is_bwd = 1) call of
 * these sizes would run under the schedule setting in force: one entry per
 * launch group (roles sharing (d, e) run in one launch; the backward with
 * d != e has two groups).  Host-only, launches nothing.  Fills up to max_out
 * entries of `out` (which may be NULL) and returns the number of groups, 0
 * for an empty problem or fp32 inputs (one SIMT launch, no plan), or -1 for
 * arguments the calls would reject.
 */
typedef struct {
    int d, e;                  /* operand widths of the group's roles (a, b: d; c: e) */
    int schedule;              /* LA2_SCHEDULE_UNIFORM or LA2_SCHEDULE_BALANCED */
    long long units;           /* (sequence, role) units: B * H * roles in the group */
    int segments;              /* UNIFORM: segments each unit is cut into; BALANCED: 0 */
    int tiles_per_cta;         /* 128-position tiles of a segment (UNIFORM, the last may be
                                  shorter) or of a CTA's run (BALANCED) */
    long long ctas;            /* CTAs of the scan launch */
    long long prepass_ctas;    /* CTAs of the state pre-pass launch (0: no pre-pass) */
} la2_plan;

int la2_plan_info(int B, int H, int T, int d, int e, int block, la2_dtype dtype, int is_bwd,
                  la2_plan *out, int max_out);

/*
 * Forward: out[b,h,t,:] = sum_{s<=t} decay[h]^(t-s) (q[b,h,t,:] . k[b,h,s,:]) v[b,h,s,:].
 *
 * Supported: dtype F32 with 1 <= d, e <= 128 and any block; dtype BF16 with
 * d, e in {64, 128} and any block.  Anything else well-formed returns
 * LA2_ERR_UNSUPPORTED.  On the BF16 path block = 128 runs the warp-specialised
 * tcgen05 kernel (the fast path: overlapped pipeline, sequences cut into
 * segments to fill the GPU); block = 64 and 256 run a phase-serial tcgen05
 * kernel with the state carried across 64- or 256-row blocks in fp32
 * registers (one CTA per sequence and 64 value columns, no segments; carried
 * states and the normalised form as with block = 128).  out must not alias an input.  workspace: device
 * memory, 256-byte aligned, of at least la2_workspace_bytes(..., 0) bytes
 * (LA2_ERR_WORKSPACE otherwise), not used concurrently by another call.
 */
la2_status la2_fwd(const void *q, const void *k, const void *v, const float *decay,
                   void *out, int B, int H, int T, int d, int e, int block,
                   la2_dtype dtype, void *workspace, size_t workspace_bytes,
                   la2_stream_t stream);

/*
 * Forward with a carried state: as la2_fwd, but the recurrence starts from
 * init_state instead of zero and the state after the last position is written
 * to final_state.  With S_{-1} = init_state and S_t = decay[h] S_{t-1} +
 * k_t v_t^T (d x e), out[t] = S_t^T q_t, i.e.
 *
 *   out[b,h,t,:] = decay[h]^(t+1) init_state[b,h]^T q[b,h,t,:]
 *                  + sum_{s<=t} decay[h]^(t-s) (q[b,h,t,:] . k[b,h,s,:]) v[b,h,s,:]
 *   final_state[b,h] = S_{T-1}
 *
 * The state is everything a sequence carries from one position to the next
 * ("Lightning Attention" explainer, section 2, memory footprint), so a long
 * sequence can be processed in consecutive pieces, each starting from the
 * final state of the one before, with the result of one call over the whole.
 *
 * init_state, final_state: device fp32 [B, H, d, e] contiguous (row i = key
 * feature, column j = value feature), 4-byte aligned; either may be NULL
 * (start from zero / do not write the state).  final_state must not alias
 * init_state or any other argument.  With T = 0 the final state is the
 * initial one (or zero).  Support matrix and workspace as for la2_fwd.
 */
la2_status la2_fwd_state(const void *q, const void *k, const void *v, const float *decay,
                         void *out, const float *init_state, float *final_state,
                         int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                         void *workspace, size_t workspace_bytes, la2_stream_t stream);

/*
 * la2_fwd_state with an explicit layout of q, k, v and out (see la2_layout)
 * and an output element type out_dtype (F32, or BF16 with BF16 inputs; see
 * la2_dtype); everything else as la2_fwd_state.  The states stay fp32.  An
 * unknown layout or out_dtype is LA2_ERR_INVALID_ARG.
 */
la2_status la2_fwd_ex(const void *q, const void *k, const void *v, const float *decay,
                      void *out, const float *init_state, float *final_state,
                      int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                      la2_dtype out_dtype, la2_layout layout, void *workspace,
                      size_t workspace_bytes, la2_stream_t stream);

/*
 * Backward of L = sum dout * out with respect to q, k and v (decay is not
 * differentiated):
 *   dq[t] = sum_{s<=t} lambda^(t-s) (dout_t . v_s) k_s
 *   dk[s] = sum_{t>=s} lambda^(t-s) (v_s . dout_t) q_t
 *   dv[s] = sum_{t>=s} lambda^(t-s) (k_s . q_t) dout_t
 * Nothing is saved by la2_fwd; the backward recomputes what it needs.  Same
 * support matrix as la2_fwd.  dq, dk, dv must not alias each other or an
 * input.
 */
la2_status la2_bwd(const void *q, const void *k, const void *v, const float *decay,
                   const void *dout, void *dq, void *dk, void *dv,
                   int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                   void *workspace, size_t workspace_bytes, la2_stream_t stream);

/*
 * One recurrent decode step: one new token per sequence (b, h).
 *
 *   state[b,h] <- decay[h] state[b,h] + k[b,h,:] v[b,h,:]^T     (d x e, in place)
 *   out[b,h,:]  = state[b,h]^T q[b,h,:]                         (with the new state)
 *
 * This is the prefix-sum recurrence of the "Lightning Attention" explainer
 * (section 1) advanced by one position; starting from the final state of
 * la2_fwd_state over a prompt, successive calls continue the same sequence at a
 * constant cost per token (the Lightning Attention-2 abstract's constant speed).
 *
 * q, k: device [B, H, d] of `dtype`; v: device [B, H, e] of `dtype` (element
 * aligned); decay: device fp32 [H]; state: device fp32 [B, H, d, e] contiguous,
 * 4-byte aligned (16-byte aligned with e % 4 == 0 takes the vector path), read
 * and written; out: device fp32 [B, H, e].  out must not alias state or an
 * input.  1 <= d, e <= 4096; B = 0 or H = 0 is empty (LA2_OK, nothing
 * launched).  Asynchronous on `stream`, one launch.
 */
la2_status la2_decode(const void *q, const void *k, const void *v, const float *decay,
                      float *state, float *out, int B, int H, int d, int e, la2_dtype dtype,
                      la2_stream_t stream);

/*
 * la2_bwd with an explicit layout of q, k, v, dout, dq, dk and dv (see
 * la2_layout) and the element type out_dtype of dq, dk and dv (as in
 * la2_fwd_ex); everything else as la2_bwd.
 */
la2_status la2_bwd_ex(const void *q, const void *k, const void *v, const float *decay,
                      const void *dout, void *dq, void *dk, void *dv,
                      int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                      la2_dtype out_dtype, la2_layout layout, void *workspace,
                      size_t workspace_bytes, la2_stream_t stream);

/*
 * Backward with carried states: the gradients of
 *
 *     L = sum_t dout_t . out_t + <d_final_state, S_{T-1}>
 *
 * for the forward of la2_fwd_state started from init_state (S_{-1}), with
 * respect to q, k, v and init_state.  d_final_state is the gradient arriving
 * at the forward's final state from what follows (the next piece of a
 * sequence trained in pieces).  With S0 = init_state and G = d_final_state:
 *
 *   dq[t]  = sum_{s<=t} lambda^(t-s) (dout_t . v_s) k_s + lambda^(t+1) S0 dout_t
 *   dk[s]  = sum_{t>=s} lambda^(t-s) (v_s . dout_t) q_t + lambda^(T-1-s) G v_s
 *   dv[s]  = sum_{t>=s} lambda^(t-s) (k_s . q_t) dout_t + lambda^(T-1-s) G^T k_s
 *   d_init_state = sum_t lambda^(t+1) q_t dout_t^T + lambda^T G
 *
 * The state is all a piece of a sequence carries ("Lightning Attention"
 * explainer, section 2, memory footprint): the backward of the last piece
 * from the incoming state, then of each earlier piece with the d_init_state
 * of the one after it as its d_final_state, gives the gradients of the whole.
 *
 * init_state, d_final_state: device fp32 [B, H, d, e], or NULL (zero);
 * d_init_state: device fp32 [B, H, d, e], or NULL (not computed); all 4-byte
 * aligned, d_init_state aliasing nothing else.  With T = 0, d_init_state =
 * d_final_state.  Layout, out_dtype (of dq, dk, dv; d_init_state stays
 * fp32), support matrix and workspace as la2_bwd_ex (the same size with or
 * without states).
 */
la2_status la2_bwd_state(const void *q, const void *k, const void *v, const float *decay,
                         const void *dout, const float *init_state, const float *d_final_state,
                         void *dq, void *dk, void *dv, float *d_init_state,
                         int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                         la2_dtype out_dtype, la2_layout layout, void *workspace,
                         size_t workspace_bytes, la2_stream_t stream);

/*
 * Gradient with respect to the decay: d_decay[h] = sum over the batch of
 * dL/dlambda_h, for the same L as la2_bwd_state (the forward from init_state,
 * d_final_state the gradient arriving at its final state; NULL = zero):
 *
 *   dL/dlambda = sum_{s<t} (t-s) lambda^(t-s-1) (q_t . k_s)(dout_t . v_s)
 *                + sum_t (t+1) lambda^t q_t^T S0 dout_t + <G, dS_{T-1}/dlambda>
 *
 * i.e. the recurrence of the "Lightning Attention" explainer (section 1) with
 * its decay differentiated: U_t = dS_t/dlambda = lambda U_{t-1} + S_{t-1}, and
 * dL/dlambda = sum_t q_t^T U_t dout_t + <G, U_{T-1}>.  The pages print no
 * gradient in lambda; this is the derivative of the definition.
 *
 * Inputs as la2_bwd_state (dtype F32 or BF16, any 1 <= d, e <= 128, both
 * layouts, element-aligned pointers); d_decay: device fp32 [H], overwritten.
 * Computed in fp32 SIMT arithmetic with the scalar accumulated in fp64, in 32-
 * row sub-tiles, each sequence cut into up to 32 segments (a pre-pass gives
 * each segment its incoming states); the batch is summed in a fixed order, so
 * the result is deterministic.  workspace: device memory of at least
 * la2_dlambda_workspace_bytes() bytes, 256-byte aligned (LA2_ERR_WORKSPACE if
 * missing or short), flat in T.  B = 0 or T = 0 writes zeros.  Asynchronous on
 * `stream`; two or three launches.
 */
size_t la2_dlambda_workspace_bytes(int B, int H, int T, int d, int e, la2_dtype dtype);

la2_status la2_dlambda(const void *q, const void *k, const void *v, const float *decay,
                       const void *dout, const float *init_state, const float *d_final_state,
                       float *d_decay, int B, int H, int T, int d, int e, la2_dtype dtype,
                       la2_layout layout, void *workspace, size_t workspace_bytes,
                       la2_stream_t stream);

/*
 * The normalised form.  The "Lightning Attention" explainer (section 1) writes
 * causal linear attention with a denominator, and (section 2) runs its
 * running sum z as a recurrence parallel to the state.  With the identity
 * feature map (the explainer's default; any other feature map phi is applied to
 * q and k by the caller before the call, since the tiling does not depend on
 * it) and the decay on both sums:
 *
 *   z_t = lambda z_{t-1} + k_t,   den_t = q_t . z_t,
 *   y_t = (sum_{s<=t} lambda^(t-s) (q_t . k_s) v_s) / den_t
 *
 * la2_fwd_norm writes y (fp32, the layout of v) and, unless den is NULL, den
 * (fp32 [B, H, T]).  la2_bwd_norm takes y and den from the forward and dy (the
 * gradient of y, the input dtype, the layout of v) and writes dq, dk, dv
 * (fp32):
 *
 *   dnum_t = dy_t / den_t,   dden_t = -(dy_t . y_t) / den_t,
 *   dq_t = sum_{s<=t} lambda^(t-s) (dnum_t . v_s) k_s + dden_t z_t,
 *   dk_s = sum_{t>=s} lambda^(t-s) (v_s . dnum_t) q_t + sum_{t>=s} lambda^(t-s) dden_t q_t,
 *   dv_s = sum_{t>=s} lambda^(t-s) (k_s . q_t) dnum_t.
 *
 * dnum enters the tensor-core scans without being rounded to the input type:
 * the dk and dv scans weigh their summed position t by 1/den_t in fp32 (in
 * their masks and state updates), and the dq scan's rows are divided by den_t
 * afterwards.  This matters because dq and dk are each the difference of two
 * nearly equal parts when y depends weakly on q and k.  The sums over
 * positions of d-vectors (z, and the dk term in dden) are SIMT scans.
 *
 * The caller keeps den_t away from zero (e.g. with a positive feature map);
 * nothing is checked.  Support as la2_fwd (d <= 128 for both dtypes' paths),
 * both layouts.  workspace: at least la2_norm_workspace_bytes(..., is_bwd)
 * bytes, 256-byte aligned; the backward's grows with T (two fp32 values per
 * position: dden and 1/den).  Asynchronous on `stream`.
 */
size_t la2_norm_workspace_bytes(int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                                int is_bwd);

la2_status la2_fwd_norm(const void *q, const void *k, const void *v, const float *decay,
                        float *y, float *den, int B, int H, int T, int d, int e, int block,
                        la2_dtype dtype, la2_layout layout, void *workspace,
                        size_t workspace_bytes, la2_stream_t stream);

la2_status la2_bwd_norm(const void *q, const void *k, const void *v, const float *decay,
                        const float *y, const float *den, const void *dy, void *dq, void *dk,
                        void *dv, int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                        la2_layout layout, void *workspace, size_t workspace_bytes,
                        la2_stream_t stream);

/* Static, human-readable name of a status code. */
const char *la2_status_str(la2_status status);

/*
 * Reads (and, if reset != 0, clears) the device status word of the current
 * device: 0 when no kernel has reported a fault, otherwise a code whose low
 * byte is the la2_status value and whose upper bits say where the kernel gave
 * up.  Synchronises with the device.  Returns LA2_ERR_CUDA if the read fails.
 */
la2_status la2_device_status(int *code, int reset);

/* Number of kernel launches the last successful la2_fwd / la2_bwd call made
 * on this host thread. */
int la2_last_launch_count(void);

/*
 * Self-test of the failure path of the bf16 scan kernel (no counterpart in
 * the paper).  Launches the forward kernel once on one sequence (B = H = 1,
 * 1 <= T <= 256, d, e in {64, 128}, block 128, bf16, [B, H, T, D]) with its
 * producer first waiting on a device flag that nothing ever sets, bounded by
 * limit_us microseconds (1 .. 1,000,000).  The wait runs out before any load
 * is issued; the kernel records LA2_ERR_TIMEOUT | (90 << 8) in the device
 * status word, every role leaves its loop through the CTA's abort flag, the
 * kernel frees its TMEM and returns, and the context stays usable.  `out` is
 * not written.  Returns LA2_OK once the launch is queued; read the recorded
 * code with la2_device_status.  Nothing traps, faults or hangs.
 */
la2_status la2_selftest_timeout(const void *q, const void *k, const void *v, const float *decay,
                                void *out, int T, int d, int e, unsigned limit_us,
                                la2_stream_t stream);

/*
 * la2_fwd without a workspace argument, for callers that cannot allocate
 * device memory at call time: code running inside CUDA-graph capture, under a
 * framework that owns every allocation, or in a context where cudaMalloc is
 * not allowed.  (No counterpart in the paper; this is a deployment variant of
 * la2_fwd.)  The inputs and the output are still the caller's; the scratch
 * la2_fwd would take from the workspace (per-segment states, when few
 * sequences are cut into segments) comes from an array built into the
 * library: kStaticScratchBytes = 148 * 128 * 128 * 4 bytes (9.25 MiB), which
 * every GPU that loads the library keeps until the process exits.  Every
 * forward call fits in it; larger requirements would return
 * LA2_ERR_WORKSPACE.  Nothing is allocated or freed.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call outside any stream
 * capture.  All calls share the one array and it keeps whatever the last call
 * left there (each call writes every value it later reads), so calls that
 * overlap on the GPU -- on different streams, or concurrently from several
 * threads -- race and must not be issued.  Results are those of la2_fwd.
 */
la2_status la2_fwd_noalloc(const void *q, const void *k, const void *v, const float *decay,
                           void *out, int B, int H, int T, int d, int e, int block,
                           la2_dtype dtype, la2_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LA2_H_ */
