/*
 * m3.h -- C ABI of the Mamba-3 mixer hot path on B200 (sm_100a).
 *
 * The library computes the Mamba-3 SSM recurrence (Mamba-3 paper summary,
 * "Technical Approach"):
 *
 *   Proposition 1 (exponential-trapezoidal discretisation):
 *     h_t = alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1}^T + gamma_t B_t x_t^T,
 *     alpha_t = exp(dt_t A_t), beta_t = (1 - lam_t) dt_t alpha_t, gamma_t = lam_t dt_t
 *   Propositions 2-4 (complex-valued transition as a data-dependent rotation):
 *     every state pair (2i, 2i+1) is rotated by dt_t theta_t[i] each step, and the
 *     left-endpoint (beta) term is rotated with the previous state, so in the
 *     original frame  h_t = R_t (alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1}^T)
 *                          + gamma_t B_t x_t^T
 *   MIMO ("Multi-Input, Multi-Output Formulation"): B_t, C_t are N x R and x_t is
 *     P x R; the input term is a rank-R sum and the readout is P x R:
 *     Y_t = h_t^T C_t + D x_t   (D is a per-head scalar skip; SISO is R = 1)
 *   Optional fused parts (m3_extras, the *_ex and *_gated entry points): the output
 *     gate y * SiLU(z), BCNorm with head-specific BC biases on B and C, and the MIMO
 *     lightweight expansion of x and z from P to P x R values per head.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no device memory and never synchronises the stream, except in
 *     m3_query_status.  Calls are asynchronous and ordered on `stream` (a
 *     cudaStream_t passed as void*; NULL is the legacy default stream).
 *   - Row-major layouts, last index contiguous:
 *       x, y        [batch][T][H][R][P]     io dtype
 *       B, C        [batch][T][G][R][N]     io dtype   (shared by the H/G heads of a group)
 *       dt, A, lam  [batch][T][H]           float      (dt after softplus, lam after sigmoid)
 *       theta       [batch][T][G][N/2]      float      (angle per state pair; see flags)
 *       D           [H]                     float      (may be NULL: no skip term)
 *       state.h     [batch][H][N][P]        float      (original frame)
 *       state.x_prev[batch][H][R][P]        io dtype   (previous token's x)
 *       state.B_prev[batch][G][R][N]        io dtype   (previous token's B)
 *     Head h reads group g = h / (H/G).  The decode step drops the T axis.
 *     State pair i is stored interleaved at rows (2i, 2i+1).
 *   - Errors: arguments are validated on the host before anything is launched;
 *     a failed check returns a status code and touches no memory.  Device code
 *     never traps; a bounded device-side wait that gives up writes
 *     M3_ERR_TIMEOUT into the workspace status word (see m3_query_status).
 *   - Value ranges are the caller's contract: dt > 0, A <= 0, lam in [0, 1].
 *     M3_FLAG_DEBUG_CHECKS adds a non-trapping device scan of them.
 *   - Tensor memory: the tensor-core kernels (bf16 prefill, chunked backward) size their
 *     tensor-memory columns so that the CTAs one kernel places on an SM fit in its 512
 *     columns together (prefill 512 x 1, backward 128 x 4 and 256 x 2).  Calls ordered on one
 *     stream never share an SM's tensor memory.  Running them concurrently on several
 *     streams, or beside other kernels that allocate tensor memory, is not supported.
 */
#ifndef M3_H
#define M3_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    M3_OK = 0,
    M3_ERR_NULL = 1,        /* a required pointer is NULL */
    M3_ERR_SHAPE = 2,       /* dims / seqlen / chunk out of range or inconsistent */
    M3_ERR_DTYPE = 3,       /* unknown io dtype */
    M3_ERR_ALIGN = 4,       /* a pointer is not aligned as documented */
    M3_ERR_UNSUPPORTED = 5, /* valid arguments that no kernel of this build handles */
    M3_ERR_WORKSPACE = 6,   /* workspace missing, misaligned or below its minimum size */
    M3_ERR_LAUNCH = 7,      /* a kernel launch failed (cudaGetLastError) */
    M3_ERR_TIMEOUT = 8,     /* a bounded device-side wait gave up (reported by m3_query_status) */
    M3_ERR_CUDA = 9,        /* another CUDA runtime call failed */
    M3_ERR_RANGE = 10       /* M3_FLAG_DEBUG_CHECKS found an input outside its range
                               (reported by m3_query_status) */
} m3_status;

typedef enum { M3_F32 = 0, M3_BF16 = 1 } m3_dtype;

/* Problem dimensions.  batch >= 1, H % G == 0, N even.  io_dtype is an m3_dtype. */
typedef struct {
    int32_t batch;     /* b */
    int32_t nheads;    /* H */
    int32_t ngroups;   /* G: B, C and theta are shared by H/G heads */
    int32_t headdim;   /* P */
    int32_t dstate;    /* N (even: N/2 complex state pairs) */
    int32_t rank;      /* R: 1 = SISO, > 1 = MIMO */
    int32_t io_dtype;  /* m3_dtype of x, B, C, y, x_prev, B_prev */
} m3_dims;

/* Resumable recurrent state (caller-owned device memory, layouts above).
 * h must be 16-byte aligned; x_prev and B_prev 16-byte aligned. */
typedef struct {
    float* h;
    void* x_prev;
    void* B_prev;
} m3_state;

/* Flags (bitwise OR). */
#define M3_FLAG_THETA_IS_ANGLE 1u  /* theta already holds the per-step angle: the dt multiply is skipped */
#define M3_FLAG_FORCE_SIMT 2u      /* m3_scan_fwd: run the sequential fp32 CUDA-core kernel */
/* Test hook for the failure path: the tensor-core prefill's MMA warp (and, in m3_scan_bwd's
 * chunked tensor-core path, the chunk-gradient kernel's issuing thread, before it issues
 * anything) waits on a barrier that nothing completes, with a 50 ms limit instead of 2 s.
 * The bounded wait gives up, the kernel aborts cleanly (outputs are invalid), and
 * m3_query_status reports M3_ERR_TIMEOUT; the CUDA context stays usable. */
#define M3_FLAG_TEST_STALL 4u
/* Debug scan of the caller's value ranges (m3_scan_fwd and its variants, m3_scan_bwd): one
 * extra kernel reads every input of the call once before the call runs and checks
 * dt > 0, A <= 0, lam in [0, 1] ("Technical Approach", Proposition 1: dt after softplus,
 * alpha = exp(dt A) <= 1, lam after sigmoid) and that every other value (x, B, C, theta,
 * D, z, the state) is finite.  It never traps and changes nothing: a violation sets a bit
 * in the workspace status word, which m3_query_status reports as M3_ERR_RANGE (a timeout
 * takes precedence).  The call itself still runs, on whatever it was given.  The decode
 * step has no workspace to report into: it rejects this flag with M3_ERR_UNSUPPORTED. */
#define M3_FLAG_DEBUG_CHECKS 8u

/* Bytes of each state buffer for `dims`.  Any out-pointer may be NULL. */
m3_status m3_state_bytes(const m3_dims* dims, size_t* h_bytes, size_t* x_prev_bytes,
                         size_t* B_prev_bytes);

/* Start a fresh sequence: h <- h0 (or 0 when h0 is NULL), x_prev <- 0, B_prev <- 0.
 * A fresh sequence has no previous token, so its first step has no beta term
 * (the unrolling starts from h_0 = gamma_0 B_0 x_0, "Parallel representation
 * under SSD").  h0, when given, is a device pointer in the state.h layout. */
m3_status m3_state_init(const m3_dims* dims, m3_state* state, const float* h0, void* stream);

/*
 * Optional parts of the Mamba-3 block fused into the recurrence kernels; a NULL
 * m3_extras* (or an all-zero one) means none of them.
 *
 *   z           output gate ("Technical Approach", output gating): y <- y * SiLU(z) after
 *               the skip.  Layout and io dtype of y, 16-byte aligned; NULL: no gate.
 *   B_bias,     BC biases ("Technical Approach", BC biases): head-specific, channel-wise,
 *   C_bias      [H][N] fp32, added to every rank column of B (and of the carried B_prev)
 *               and of C; NULL: no bias.
 *   bc_norm_eps BCNorm ("Technical Approach", BC normalisation): > 0 scales each token's
 *               B and C rank columns (and B_prev's) to unit RMS over N before the bias,
 *               v / sqrt(mean_n v^2 + eps); 0: off; negative or NaN: M3_ERR_SHAPE.
 *   x_expand    MIMO lightweight expansion of the input ("Multi-Input, Multi-Output (MIMO)
 *               Formulation", MIMO Parameterization Choices): [H][R][P] fp32, 16-byte
 *               aligned, a data-independent per-head vector.  When set, x holds one value
 *               per head channel, [b][T][H][P] (decode [b][H][P]), and the recurrence uses
 *               X[r][p] = x[p] * x_expand[h][r][p], rounded to the io dtype (the value an
 *               expanded io-dtype x would hold).  NULL: x is [..][H][R][P] as stated above.
 *   z_expand    the same for the gate: z is [b][T][H][P] (decode [b][H][P]) and the gate
 *               uses Z[r][p] = z[p] * z_expand[h][r][p], rounded to the io dtype.  Needs z
 *               (M3_ERR_NULL without it).  NULL: z has the layout of y.
 *
 * The state keeps the raw previous-token B; the map is applied wherever it is used.  With
 * x_expand, state.x_prev holds the expanded previous token X [b][H][R][P], so a state
 * moves unchanged between expanded and unexpanded calls.  y is always [..][H][R][P].
 */
typedef struct {
    const void* z;
    const float* B_bias;
    const float* C_bias;
    float bc_norm_eps;
    const float* x_expand;
    const float* z_expand;
} m3_extras;

/* Workspace bytes m3_scan_fwd uses for (dims, seqlen, chunk); at least 256
 * (the status word).  The workspace is caller-owned device memory, 256-byte
 * aligned, and must not be shared by calls that can overlap on the GPU.
 * Where batch * nheads is at most a third of the SMs of the current device (long
 * sequences with few streams, such as batch 1 x 32 heads), the bf16 tensor-core path
 * splits each sequence into segments run side by side ("Parallel representation under SSD": the carried
 * state is affine in the state entering a segment, so segments compose), and the size
 * includes their records: per (batch, head, segment) two N x P fp32 states, the
 * segment's decay and N/2 angles.  A workspace of at least the minimum (256 bytes, plus
 * the BCNorm scales of m3_scan_workspace_bytes_ex) but without room for the records is
 * accepted: the call then runs unsegmented, with the same results up to rounding.
 * Layout: [status 256][BCNorm scales][segment records]. */
m3_status m3_scan_workspace_bytes(const m3_dims* dims, int32_t seqlen, int32_t chunk,
                                  size_t* bytes);

/* Workspace bytes of m3_scan_fwd_ex with these extras: the above plus, when BCNorm is on,
 * one float per B, C and B_prev rank column of the call (its scales; 256-byte rounded). */
m3_status m3_scan_workspace_bytes_ex(const m3_dims* dims, int32_t seqlen, int32_t chunk,
                                     const m3_extras* extras, size_t* bytes);

/*
 * Prefill: run `seqlen` tokens of the recurrence for every (batch, head),
 * chunked parallel scan ("Parallel representation under SSD": the parallel
 * masked form inside a chunk of `chunk` tokens, the recurrence across chunks).
 *
 *   in : x, B, C (io dtype), dt, A, lam, theta, D (float), state (h, x_prev, B_prev)
 *   out: y [b][T][H][R][P] io dtype (rounded to nearest even from fp32);
 *        state updated in place to the end of the sequence: h = h_T (original
 *        frame), x_prev = x_{T-1}, B_prev = B_{T-1}.
 *
 * chunk must be 16, 32, 64 or 128; it only changes rounding, not the result.
 * Pointers to x, B, C, y, state buffers and the workspace must be 16-byte
 * aligned; float arrays 4-byte aligned.  seqlen == 0 is a no-op returning M3_OK
 * (only dims, chunk and the state are validated; no other pointer is examined).
 * bf16 io runs on the tcgen05 tensor-core kernel where the shape is supported
 * (P = 64, nheads % 4 == 0, and N in {64, 128} for R = 1, N = 64 for R in {2, 4});
 * other shapes and fp32 io run the sequential fp32 CUDA-core kernel.  The
 * tensor-core kernel tiles chunk * R (token, rank) rows per chunk, 64 or 128 of
 * them: a chunk whose chunk * R falls outside [64, 128] runs as the nearest tile
 * (e.g. R = 4 with chunk 64 as 32-token tiles; "Multi-Input, Multi-Output
 * Formulation" likewise shrinks the MIMO chunk by R to hold the intra-chunk
 * FLOPs), which again changes rounding only.
 */
m3_status m3_scan_fwd(const m3_dims* dims, int32_t seqlen, int32_t chunk, const void* x,
                      const void* B, const void* C, const float* dt, const float* A,
                      const float* lam, const float* theta, const float* D, m3_state* state,
                      void* y, void* workspace, size_t workspace_bytes, uint32_t flags,
                      void* stream);

/*
 * Prefill with the optional fused parts of m3_extras (extras may be NULL).  With BCNorm
 * the call first launches a small kernel for the column scales (workspace, see
 * m3_scan_workspace_bytes_ex).  Everything else is as for m3_scan_fwd.
 */
m3_status m3_scan_fwd_ex(const m3_dims* dims, int32_t seqlen, int32_t chunk, const void* x,
                         const void* B, const void* C, const float* dt, const float* A,
                         const float* lam, const float* theta, const float* D,
                         const m3_extras* extras, m3_state* state, void* y, void* workspace,
                         size_t workspace_bytes, uint32_t flags, void* stream);

/*
 * Prefill with the fused output gate ("Technical Approach", output gating: the readout
 * y_t, skip included, is multiplied element-wise by SiLU(z_t) = z_t / (1 + e^-z_t)).
 *
 *   z: [b][T][H][R][P] in the io dtype (the layout of y), device pointer, 16-byte
 *      aligned, read only.  NULL returns M3_ERR_NULL (unless seqlen == 0).
 *
 * Everything else -- arguments, state update, kernel choice, errors -- is as for
 * m3_scan_fwd; the gate changes y only, never the state.
 */
m3_status m3_scan_fwd_gated(const m3_dims* dims, int32_t seqlen, int32_t chunk, const void* x,
                            const void* B, const void* C, const float* dt, const float* A,
                            const float* lam, const float* theta, const float* D,
                            const void* z, m3_state* state, void* y, void* workspace,
                            size_t workspace_bytes, uint32_t flags, void* stream);

/*
 * Prefill without a workspace argument, for callers that cannot allocate device
 * memory (for example a plugin inside a host framework whose caching allocator owns
 * all of the device memory, or a serving loop that must not call cudaMalloc because
 * it can synchronise the device).  The pages describe no such entry point; this is a
 * deployment convenience of this library.
 *
 * Same arguments, layouts, results and errors as m3_scan_fwd, minus the workspace.
 * Every host-side check of m3_scan_fwd runs first, before any CUDA call.  The workspace
 * is lent from one fixed scratch array compiled into the library (64 KiB, 256-byte
 * aligned, held on every GPU that loads the library until the process exits), which
 * holds the status word: the call runs without sequence segments, as m3_scan_fwd does
 * with a workspace of that size.  Shapes whose minimum workspace exceeded 64 KiB would
 * be rejected with M3_ERR_WORKSPACE (none does: without extras the minimum is 256 B).
 * Nothing is allocated: no cudaMalloc / cudaFree and no allocating library routine.
 *   - `stream` must belong to the current device (the array's address is per device);
 *     a stream of another device is rejected with M3_ERR_UNSUPPORTED.
 *   - Each call looks up the array's device address on the current device.  The first
 *     call on a device loads it there: make that first call before any stream capture.
 *     The lookup is not cached, so a device reset between calls does no harm.
 *   - Every call shares the one array, and each call clears the part that must start at
 *     zero.  Calls that can overlap on the GPU (different streams without ordering) race
 *     on it: order them.
 *   - The device-side status word lives in the shared array and is not reported.  A call
 *     whose bounded device-side wait gave up (see m3_query_status) leaves y and the state
 *     undefined without saying so; callers that need to know use m3_scan_fwd with their
 *     own workspace and m3_query_status.  For the same reason M3_FLAG_DEBUG_CHECKS is
 *     rejected here with M3_ERR_UNSUPPORTED.
 */
m3_status m3_scan_fwd_noalloc(const m3_dims* dims, int32_t seqlen, int32_t chunk, const void* x,
                              const void* B, const void* C, const float* dt, const float* A,
                              const float* lam, const float* theta, const float* D,
                              m3_state* state, void* y, uint32_t flags, void* stream);

/*
 * Decode: one token of the recurrence for every (batch, head), fused in one
 * pass over the fp32 state ("Multi-Input, Multi-Output Formulation", SISO/MIMO
 * decode step, with the trapezoid and rotation of Propositions 1 and 4).
 *
 *   in : x [b][H][R][P], B, C [b][G][R][N] (io dtype), dt, A, lam [b][H],
 *        theta [b][G][N/2], D [H] (may be NULL), state
 *   out: y [b][H][R][P] io dtype; state updated in place (h, x_prev <- x,
 *        B_prev <- B).
 *
 * Supported: N even <= 256, P % 4 == 0 and P <= 256, R <= 8.
 */
m3_status m3_decode_step(const m3_dims* dims, const void* x, const void* B, const void* C,
                         const float* dt, const float* A, const float* lam,
                         const float* theta, const float* D, m3_state* state, void* y,
                         uint32_t flags, void* stream);

/* Decode step with the optional fused parts of m3_extras (z [b][H][R][P]); BCNorm scales
 * are computed inside the kernel.  Otherwise as m3_decode_step. */
m3_status m3_decode_step_ex(const m3_dims* dims, const void* x, const void* B, const void* C,
                            const float* dt, const float* A, const float* lam,
                            const float* theta, const float* D, const m3_extras* extras,
                            m3_state* state, void* y, uint32_t flags, void* stream);

/*
 * Decode step with the fused output gate: y = (h^T C + D x) * SiLU(z), z [b][H][R][P] in
 * the io dtype, 16-byte aligned, not NULL (M3_ERR_NULL).  Otherwise as m3_decode_step.
 */
m3_status m3_decode_step_gated(const m3_dims* dims, const void* x, const void* B, const void* C,
                               const float* dt, const float* A, const float* lam,
                               const float* theta, const float* D, const void* z,
                               m3_state* state, void* y, uint32_t flags, void* stream);

/*
 * Backward pass of m3_scan_fwd (without extras): the reverse-mode gradients of a scalar loss
 * L given dL/dy and dL/dh_T.  The pages describe only the forward recurrence; this is its
 * derivative, taken token by token in reverse through the same operations (Proposition 1
 * with the rotation of Propositions 2 and 4; MIMO rank-R input and readout):
 *   Lam = dL/dh_t:  Lam += C dy^T;  dC = h_t dy^T;  dx = D dy + gamma B^T Lam (+ beta B^T dM of
 *   the next token);  dB = gamma Lam x^T (+ beta dM x^T of the next token);  dM = R(phi)^T Lam;
 *   Lam <- alpha dM;  and through alpha = e^{dt A}, beta = (1 - lam) dt alpha, gamma = lam dt,
 *   phi = dt theta to ddt, dA, dlam, dtheta.
 *
 *   in : the forward call's inputs x, B, C (io dtype), dt, A, lam, theta, D (may be NULL);
 *        state0: the state that forward call STARTED from (h0, x_prev, B_prev; read only);
 *        dy [b][T][H][R][P] io dtype; dhT [b][H][N][P] fp32 or NULL (zero).
 *   out: grads (fp32, caller-owned, overwritten, not NULL except dD):
 *        dx [b][T][H][R][P]; dB, dC [b][T][G][R][N] and dtheta [b][T][G][N/2], each summed
 *        over the heads of its group; ddt, dA, dlam [b][T][H]; dD [H] summed over batch and
 *        tokens (ignored when D is NULL; may be NULL); dh0 [b][H][N][P]; dx_prev [b][H][R][P];
 *        dB_prev [b][G][R][N] (summed over the group's heads).
 *   The carried x_prev / B_prev outputs of the forward call (copies of its last token) get no
 *   gradient here: a caller chaining calls adds theirs to dx / dB of the last token.
 *   Two implementations, chosen by shape:
 *   - bf16 io, P = 64, and either R = 1 with N in {64, 128} or R in {2, 4} with N = 64 (and
 *     dx, dB, dC 16-byte aligned): the chunked backward on the tensor cores ("Parallel
 *     representation under SSD"; chunks of 64 / R tokens, 64 (token, rank) rows).  Chunk
 *     products, a scan over chunks for the entering states and leaving adjoints (stored in the
 *     workspace as bf16), the chunk gradients from bf16 operands with fp32 accumulation, and
 *     the angle carries.  dB, dC, dB_prev and dD are accumulated with atomics (last bits may
 *     vary from run to run); dtheta is summed over the group's heads in a fixed order.
 *     Accuracy: the bf16 bar of the prefill (about 1e-2 of each gradient's largest value).
 *   - every other shape, and any shape with M3_FLAG_FORCE_SIMT: a sequential fp32 kernel,
 *     one CTA per (batch, head), with the states recomputed from checkpoints every segment
 *     of up to 16 tokens, then the per-head shares of the group gradients summed in a fixed
 *     order.  The sums over state pairs inside a head use shared-memory atomics, so dx, ddt,
 *     dA and dlam may differ in the last bits from run to run.
 *   Supported: N even, N <= 256, P <= 64, R in {1, 2, 3, 4, 8}, within the sequential
 *   kernel's thread and shared-memory limits (else M3_ERR_UNSUPPORTED).  seqlen 0 does
 *   nothing.  A wait of the chunked path that runs out of time reports M3_ERR_TIMEOUT
 *   through the workspace's status word (m3_query_status).
 */
typedef struct {
    float* dx;
    float* dB;
    float* dC;
    float* ddt;
    float* dA;
    float* dlam;
    float* dtheta;
    float* dD;
    float* dh0;
    float* dx_prev;
    float* dB_prev;
} m3_grads;

/* Workspace bytes of m3_scan_bwd for (dims, seqlen): the status block, then the larger of
 * the two implementations' needs.  Sequential: per (batch, head) one N x P fp32 state per
 * segment and one segment of states, and the per-head shares of the group gradients
 * (2 R N + N/2 floats per token and head).  Chunked (the shapes listed at m3_scan_bwd): per
 * (batch, head, chunk) four N x P bf16 tiles and a few scalars per state pair, plus one
 * fp32 angle gradient per (batch, head, token, pair). */
m3_status m3_scan_bwd_workspace_bytes(const m3_dims* dims, int32_t seqlen, size_t* bytes);

m3_status m3_scan_bwd(const m3_dims* dims, int32_t seqlen, const void* x, const void* B,
                      const void* C, const float* dt, const float* A, const float* lam,
                      const float* theta, const float* D, const m3_state* state0,
                      const void* dy, const float* dhT, const m3_grads* grads, void* workspace,
                      size_t workspace_bytes, uint32_t flags, void* stream);

/* Backward pass of m3_scan_fwd_ex, the prefill with the fused extras, by the chain rule
 * around the recurrence's backward ("Technical Approach": output gating, BC normalisation,
 * BC biases; "MIMO Parameterization Choices": the lightweight expansion).  The forward is
 * the recurrence on effective inputs X = x w_x, Z = z w_z, per-head B_h = B s(B) + B_bias[h]
 * (s the BCNorm scale, 1 when off), C_h likewise, theta shared as before, followed by the
 * gate y = y_pre SiLU(Z).  The backward
 *   - forms the effective inputs (rounded to the io dtype, as the fused kernels use them);
 *   - with the gate, reruns the forward without it for y_pre (from a copy of state0) and
 *     takes dL/dy_pre = dy Z sig(Z), dL/dZ = dy y_pre sig(Z) (1 + Z (1 - sig(Z)));
 *   - runs m3_scan_bwd's recurrence backward on the effective inputs, one group per head
 *     when the BC map is on;
 *   - maps back: dx = sum_r dX w_x, dw_x = sum_{b,t} dX x (z likewise), dB = J(sum over the
 *     group's heads of dB_h) with the RMS scale's Jacobian J(du) = s du - (s^3/N) v <du, v>,
 *     dB_bias[h] = sum_{b,t,r} dB_h (plus the carried B_prev's share), C likewise.
 *   in : the forward call's inputs, state0 and extras (as given to m3_scan_fwd_ex), dy in the
 *        layout of y, dhT or NULL.
 *   out: grads as m3_scan_bwd (dx [b][T][H][P] with x_expand; dx_prev refers to the
 *        expanded x_prev the state holds); m3_extra_grads below, fp32, caller-owned,
 *        overwritten.  An extras pointer that is NULL or all zero runs m3_scan_bwd itself.
 *   The parameter gradients (dx_expand, dz_expand, dB_bias, dC_bias) and, on the chunked
 *   path, the group-shared ones are sums accumulated with atomics.  Supported: the shapes of
 *   m3_scan_bwd (its chunked tensor-core shapes run the chunked backward).
 *   Workspace: m3_scan_bwd_workspace_bytes_ex (the recurrence backward's own workspace
 *   first, then the effective inputs, their gradients and, with the gate, the forward's
 *   workspace, a state copy and y_pre). */
typedef struct {
    float* dz;         /* layout of z ([b][T][H][P] with z_expand); needed iff the gate is on */
    float* dB_bias;    /* [H][N]; needed iff B_bias */
    float* dC_bias;    /* [H][N]; needed iff C_bias */
    float* dx_expand;  /* [H][R][P]; needed iff x_expand */
    float* dz_expand;  /* [H][R][P]; needed iff z_expand */
} m3_extra_grads;

m3_status m3_scan_bwd_workspace_bytes_ex(const m3_dims* dims, int32_t seqlen,
                                         const m3_extras* extras, size_t* bytes);

m3_status m3_scan_bwd_ex(const m3_dims* dims, int32_t seqlen, const void* x, const void* B,
                         const void* C, const float* dt, const float* A, const float* lam,
                         const float* theta, const float* D, const m3_state* state0,
                         const m3_extras* extras, const void* dy, const float* dhT,
                         const m3_grads* grads, const m3_extra_grads* extra_grads,
                         void* workspace, size_t workspace_bytes, uint32_t flags, void* stream);

/* Synchronise `stream` and report the device-side status word in `workspace`:
 * M3_OK, M3_ERR_TIMEOUT when a bounded wait gave up, or M3_ERR_RANGE when the debug
 * scan of M3_FLAG_DEBUG_CHECKS found an input outside its range. */
m3_status m3_query_status(const void* workspace, void* stream);

/* Static English text for a status code. */
const char* m3_status_string(m3_status status);

#ifdef __cplusplus
}
#endif

#endif /* M3_H */
