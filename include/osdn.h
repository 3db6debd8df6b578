/*
 * osdn.h - C ABI of libosdn.so: the Online Scaled DeltaNet (OSDN) forward, its
 * backward (gradients for training) and single-token decode on NVIDIA B200
 * (sm_100a).
 *
 * Method: "OSDN: Improving Delta Rule with Provable Online Preconditioning in
 * Linear Attention" (gist.science technical summary).
 *   section 2.1: S_t = S_{t-1} + beta_t (v_t - S_{t-1} k_t) (d_t (.) k_t)^T,
 *                o_t = S_t q_t, S in R^{dv x dk}; the read/erase key is k_t,
 *                the write key is the scaled key d_t (.) k_t;
 *   section 2.2: the preconditioner step uses only k_t and beta_t;
 *   section 2.3: d_{t+1} = r_t d_t + eta beta_t (1 - beta_t <d_t, k_t^2>)
 *                k_t^2 / ||k_t||^2   (APF; r == 1 when APF is off).
 * Readings of points the pages leave open: the preconditioner step is a
 * descent step on the hypergradient surrogate; no projection follows it;
 * token t writes with d_t (d_1 = d0); ||k_t|| = 0 skips the step; no
 * normalisation or 1/sqrt(dk) scale is applied to q or k inside the op.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller (except the
 *     host buffers of osdn_fwd_host). The library never allocates device memory
 *     and never frees anything.
 *   - Layouts are row-major (last dimension contiguous), dense unless the
 *     strides of osdn_params say otherwise (forward only):
 *       q, k   [B, T, H, dk]     v, out [B, T, H, dv]
 *       beta, r [B, T, H]
 *       d (d0, final_d) [B, H, dk] fp32     S (S0, final_S) [B, H, dv, dk] fp32
 *     For osdn_step, T is absent: q, k [B, H, dk]; v, out [B, H, dv];
 *     beta, r [B, H].
 *   - q, k, v, beta, r and out share one element type (osdn_params.dtype);
 *     S and d are always fp32. Every pointer must be 16-byte aligned.
 *   - Work is enqueued on the caller's CUDA stream (cudaStream_t passed as
 *     void*, NULL = legacy default stream) and returns without a host sync.
 *   - Return value: OSDN_OK or an OSDN_ERR_* code; nothing aborts. A
 *     human-readable message for the calling thread's last error is available
 *     from osdn_get_last_error().
 *   - Supported sizes: dk, dv in {64, 128}; chunk = 64; B, H >= 1; T >= 0
 *     (T = 0 copies the initial state to the final state).
 */
#ifndef OSDN_H
#define OSDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define OSDN_ABI_VERSION 3

enum {
    OSDN_OK = 0,
    OSDN_ERR_INVALID_ARG = 1,   /* NULL required pointer, bad size, misalignment */
    OSDN_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. dk = 96) */
    OSDN_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    OSDN_ERR_TIMEOUT = 4        /* a bounded device-side wait gave up */
};

typedef enum { OSDN_BF16 = 0, OSDN_FP32 = 1 } osdn_dtype;

typedef struct {
    uint32_t struct_size;   /* must be sizeof(osdn_params): ABI versioning */
    int32_t B;              /* sequences */
    int32_t T;              /* tokens per sequence (ignored by osdn_step) */
    int32_t H;              /* heads */
    int32_t dk;             /* key / query width */
    int32_t dv;             /* value width */
    int32_t chunk;          /* chunk length C of the chunkwise form; 64 */
    int32_t dtype;          /* osdn_dtype of q, k, v, beta, r, out */
    float eta;              /* hypergradient step size of the preconditioner */
    int32_t apf_anchor;     /* 0: APF retention r d (toward 0); 1: anchored APF,
                               r d + (1 - r) d_anchor, d_anchor = d0 in the forward */
    /* Element strides of q, k, v and out over their (b, t, h) dimensions (the
     * last dimension is always contiguous). All three zero: the dense layout
     * [B, T, H, width]. Otherwise each stride must be a non-negative multiple of
     * 8 elements (16-byte rows for the tensor-memory-accelerator loads), for
     * example q, k, v read in place as column slices of one fused projection
     * [B, T, H, 2 dk + dv]. Honoured by the forward entry points (osdn_fwd and
     * its phases, the gated and no-allocation forwards); osdn_step* and osdn_bwd
     * take dense tensors only and return OSDN_ERR_UNSUPPORTED otherwise.
     * beta, r and alpha are always dense [B, T, H]. */
    int64_t stride_q[3];
    int64_t stride_k[3];
    int64_t stride_v[3];
    int64_t stride_o[3];
} osdn_params;
/* Earlier versions of this struct are accepted by struct_size: version 1
 * ended after eta (36 bytes; apf_anchor = 0), version 2 after apf_anchor
 * (40 bytes); both get the dense layout. */

/* Bytes of device workspace osdn_fwd needs for these parameters (written to
 * *bytes). The workspace holds the scaled write keys d_t (.) k_t in the input
 * dtype [B, T, H, dk] and, when phase 2 splits the sequences into segments
 * (osdn_fwd_segments > 1), three fp32 states per segment and head (start
 * state, own end state, transfer; 3 * B * P * H * dv * dk * 4 bytes) and a
 * 16 KiB tile of zeros. When osdn_fwd pipelines the scan with phase 2
 * (osdn_fwd_launches) it also holds beta, r and alpha reordered by segment
 * (3 * B * T * H * 2 bytes) and two fp32 states and two d vectors per (b, h)
 * handed from segment to segment. It is scratch owned by the caller, needs no
 * initialisation, and may be reused by the next call on the same stream. The
 * size depends on the SM count of the current device.
 * Returns OSDN_OK, OSDN_ERR_INVALID_ARG or OSDN_ERR_UNSUPPORTED. */
int osdn_fwd_workspace_size(const osdn_params *p, size_t *bytes);

/* Number of segments P that phase 2 (osdn_fwd, osdn_fwd_chunk and their gated
 * forms) cuts every sequence into, written to *segments; 1 means no split.
 * Phase 2 carries the state serially through the chunks of a sequence, so
 * with few (b, h) units most SMs would idle. On the tensor-core path (bf16,
 * dk = dv = 128, dense tensors) P is the largest power of two up to 16 with
 * B * H * P <= the SM count, lowered until T is a multiple of 64 P with
 * T / P >= 512; P < 4 is not used. One sequence (B = 1, anchored APF off)
 * with T a multiple of 1024, T >= 8192 and 3 H <= the SM count takes P = 16:
 * osdn_fwd then overlaps the scan with phase 2 (osdn_fwd_launches), where
 * short segments keep the work left after the scan short. Each chunk update is affine in the state
 * (technical summary section 2.1: S <- S (I - W^T Kw) + U0^T Kw), so a
 * segment's end state is S_start E + L, with L its end state from S = 0 and E
 * its end state from S = I with V = 0. A split call runs the chunk kernel
 * three times over the B * P segments (for L, for E, and for the outputs from
 * the combined start states) plus two small kernels (identity fill,
 * combine). The outputs equal the unsplit ones up to rounding.
 * Errors: OSDN_ERR_INVALID_ARG (bad params, NULL segments), OSDN_ERR_UNSUPPORTED. */
int osdn_fwd_segments(const osdn_params *p, int *segments);

/* Kernel launches one osdn_fwd (or osdn_fwd_gated) call makes, written to
 * *launches: 2 without segments (scan, chunk); 6 with segments (scan, identity
 * fill, three chunk passes, combine). With segments and one sequence (B = 1,
 * anchored APF off) osdn_fwd overlaps the scan with phase 2. Segments
 * 0 .. P - 2 go in batches of nb = min(P / 2, (SMs - H) / (2 H)); the scan
 * runs on cuda_stream as one launch per batch and one for the last segment,
 * each from the d the previous one ended with, while two library-owned
 * non-blocking streams (created on first use, forked from and joined back to
 * cuda_stream by events) run each batch's chunk passes as soon as the scan
 * has covered it, and the last segment's output pass after the scan:
 * 2 + 5 ceil((P - 1) / nb) launches.
 * Without segments, when B * H is at most half the SM count (tensor-core path,
 * dense tensors, anchored APF off), osdn_fwd instead pipelines the two phases
 * over Q = 4 segments of each sequence when each keeps at least 1024 tokens
 * (else 2 of at least 512, else none): one launch reorders beta, r and alpha by
 * segment, then cuda_stream scans segment after segment (each scan from the
 * d the previous one ended with) while a library-owned stream runs phase 2 of
 * each segment once it is scanned, from the state the previous segment ended
 * with: 1 + 2 Q launches, with phase 2 of segment s beside the scan of s + 1
 * on other SMs. Segments end on chunk boundaries and hand over d and S in
 * fp32, so the results equal the unpipelined ones bit for bit.
 * T = 0: at most one (d filled with ones).
 * Errors: OSDN_ERR_INVALID_ARG (bad params, NULL launches), OSDN_ERR_UNSUPPORTED. */
int osdn_fwd_launches(const osdn_params *p, int *launches);

/* Chunkwise-parallel OSDN forward over T tokens for every (b, h).
 *   Phase 1 (preconditioner scan, section 2.2 "two phases"): d_t for every
 *   token from k, beta, r and d0; the scaled write keys d_t (.) k_t go to the
 *   workspace; d after the last token goes to final_d.
 *   Phase 2 (chunked delta rule with the scaled write key, section 2.1): per
 *   chunk of C tokens, A = strict_tril(diag(beta) K Kw^T),
 *   T = (I + A)^{-1}, U = T diag(beta) (V - K S^T),
 *   O = Q S^T + tril(Q Kw^T) U, S <- S + U^T Kw (Kw = scaled write keys).
 * r == NULL: APF off (r == 1). d0 == NULL: d0 = ones. S0 == NULL: S0 = 0.
 * p->apf_anchor != 0: anchored APF, d_{t+1} = r_t d_t + (1 - r_t) d0 + (the same
 * hypergradient step), i.e. the retention pulls d toward d0 instead of 0.
 * final_S, final_d may be NULL (not written). out may not be NULL when T > 0.
 * workspace must hold osdn_fwd_workspace_size() bytes (16-byte aligned).
 * Errors: OSDN_ERR_INVALID_ARG, OSDN_ERR_UNSUPPORTED, OSDN_ERR_CUDA. */
int osdn_fwd(const osdn_params *p,
             const void *q, const void *k, const void *v,
             const void *beta, const void *r,
             const float *d0, const float *S0,
             void *out, float *final_S, float *final_d,
             void *workspace, size_t workspace_bytes,
             void *cuda_stream);

/* Phase 1 of osdn_fwd alone: the preconditioner scan. Reads k, beta, r and
 * d0; writes the scaled write keys d_t (.) k_t into the workspace and d after
 * the last token into final_d (nullable). Same arguments and rules as
 * osdn_fwd. osdn_fwd == osdn_fwd_scan then osdn_fwd_chunk on one stream. */
int osdn_fwd_scan(const osdn_params *p,
                  const void *k, const void *beta, const void *r,
                  const float *d0, float *final_d,
                  void *workspace, size_t workspace_bytes,
                  void *cuda_stream);

/* osdn_fwd_scan plus a diagnostic of the preconditioner ("OSDN: Improving
 * Delta Rule with Provable Online Preconditioning in Linear Attention",
 * technical summary sections 4-5: the contraction factor of one write):
 *   rho   [B, T, H] fp32, nullable: rho_t = (1 - beta_t <d_t, k_t^2>)^2, the
 *         factor by which token t's write shrinks its own loss,
 *         f_t(S_t) = rho_t f_t(S_{t-1}) with f_t(S) = 1/2 ||S k_t - v_t||^2;
 *         1 when the token writes nothing (beta_t = 0 or k_t = 0).
 *   q_geo [B, H] fp32, nullable: exp of the mean of log rho_t over the T tokens
 *         of each (sequence, head); 1 when T = 0, 0 when some rho_t is 0.
 * Both pointers 16-byte aligned, caller-owned. Every other argument, rule and
 * error as osdn_fwd_scan; with rho == q_geo == NULL it is osdn_fwd_scan. */
int osdn_fwd_scan_diag(const osdn_params *p,
                       const void *k, const void *beta, const void *r,
                       const float *d0, float *final_d,
                       float *rho, float *q_geo,
                       void *workspace, size_t workspace_bytes,
                       void *cuda_stream);

/* Phase 2 of osdn_fwd alone: the chunked delta rule with the scaled write
 * keys that a preceding osdn_fwd_scan with the same parameters left in the
 * workspace (ordered before this call on the stream). Writes out and
 * final_S (nullable); when it splits the sequences (osdn_fwd_segments > 1)
 * it also writes the segment scratch after the scaled keys, which it leaves
 * unchanged. Same arguments and rules as osdn_fwd. */
int osdn_fwd_chunk(const osdn_params *p,
                   const void *q, const void *k, const void *v, const void *beta,
                   const float *S0, void *out, float *final_S,
                   void *workspace, size_t workspace_bytes,
                   void *cuda_stream);

/* One recurrent decode token for every (b, h), in place (constant memory):
 *   k~ = d (.) k;  S <- S + beta (v - S k) k~^T;  out = S q (after the write);
 *   d <- r d + eta beta (1 - beta <d, k^2>) k^2 / ||k||^2 (pre-update d).
 * p->T is ignored. S [B, H, dv, dk] and d [B, H, dk] are read and written.
 * r == NULL: APF off. Errors: OSDN_ERR_INVALID_ARG, OSDN_ERR_UNSUPPORTED,
 * OSDN_ERR_CUDA. */
int osdn_step(const osdn_params *p,
              const void *q, const void *k, const void *v,
              const void *beta, const void *r,
              float *S, float *d, void *out,
              void *cuda_stream);

/* osdn_step with anchored APF (p->apf_anchor != 0): the retention step becomes
 * d <- r d + (1 - r) d_anchor + eta beta (1 - beta <d, k^2>) k^2 / ||k||^2,
 * d_anchor [B, H, dk] fp32 (NULL: ones; the d0 of the forward). With
 * p->apf_anchor == 0, d_anchor is ignored and this is osdn_step. */
int osdn_step_ex(const osdn_params *p,
                 const void *q, const void *k, const void *v,
                 const void *beta, const void *r, const float *d_anchor,
                 float *S, float *d, void *out,
                 void *cuda_stream);


/* Gated OSDN (the gated delta rule backbone the pages run OSDN on):
 *   S_t = alpha_t S_{t-1} (I - beta_t k_t kw_t^T) + beta_t v_t kw_t^T,   kw_t = d_t (.) k_t,
 * i.e. the OSDN write applied to the decayed state alpha_t S_{t-1}; the
 * preconditioner d is unchanged. alpha [B, T, H] in the input dtype, in [0, 1]
 * (alpha_t = 0 restarts the state before token t's write). The chunk form uses
 * the decay only as ratios gamma_t / gamma_j <= 1 of the cumulative gate within
 * a 64-token chunk, so every gate value in [0, 1] stays in range.
 * osdn_fwd_gated: as osdn_fwd plus alpha (not NULL when T > 0); bf16 inputs
 * with dk = dv = 128 only (else OSDN_ERR_UNSUPPORTED).
 * osdn_fwd_chunk_gated: phase 2 alone, after osdn_fwd_scan on the same stream
 * (splitting into segments as osdn_fwd_chunk does).
 * osdn_step_gated: osdn_step_ex with the decay (alpha [B, H], not NULL); every
 * dtype and width osdn_step accepts. */
int osdn_fwd_gated(const osdn_params *p,
                   const void *q, const void *k, const void *v,
                   const void *beta, const void *r, const void *alpha,
                   const float *d0, const float *S0,
                   void *out, float *final_S, float *final_d,
                   void *workspace, size_t workspace_bytes,
                   void *cuda_stream);

int osdn_fwd_chunk_gated(const osdn_params *p,
                         const void *q, const void *k, const void *v,
                         const void *beta, const void *alpha,
                         const float *S0, void *out, float *final_S,
                         void *workspace, size_t workspace_bytes,
                         void *cuda_stream);

int osdn_step_gated(const osdn_params *p,
                    const void *q, const void *k, const void *v,
                    const void *beta, const void *r, const void *alpha,
                    const float *d_anchor, float *S, float *d, void *out,
                    void *cuda_stream);

/* Backward (training). The pages give no backward pass; this is the exact
 * reverse-mode derivative of osdn_fwd (plain or anchored APF) for
 *     L = sum <dout, out> + <dS_final, final_S> + <dd_final, final_d>,
 * through both phases: the chunked delta rule with the scaled write key
 * (technical summary section 2.1) and the preconditioner recurrence of d
 * (sections 2.2-2.3), including the dependence of the write keys d_t (.) k_t
 * on k, beta, r and d0.
 * Inputs: the osdn_fwd inputs (q, k, v, beta, r, d0, S0; same layouts, same
 * NULL meanings) and the upstream gradients dout [B, T, H, dv] (input dtype),
 * dS_final [B, H, dv, dk] fp32 (NULL = 0), dd_final [B, H, dk] fp32 (NULL = 0).
 * Outputs (overwritten): dq, dk [B, T, H, dk]; dv [B, T, H, dv]; dbeta [B, T, H]
 * in the input dtype (required when T > 0); dr [B, T, H] in the input dtype
 * (written only when r and dr are both non-NULL); dd0 [B, H, dk] and
 * dS0 [B, H, dv, dk] fp32 (nullable). Under anchored APF, dd0 includes the
 * anchor's share (the anchor is d0).
 * The forward is recomputed inside the call (nothing from osdn_fwd is reused).
 * workspace: osdn_bwd_workspace_size() bytes, 16-byte aligned, no
 * initialisation needed; it holds fp32 intermediates: d_t for every token
 * (dk values) and, per 64-token chunk and head (the last chunk padded),
 * 64 * (4 dk + 3 dv + 2 * 64 + 2) values plus two states (2 dv dk values),
 * i.e. about (5 dk + 3 dv + 130) * 4 bytes per token and head plus
 * 8 dv dk bytes per chunk and head (3.5 GB at B8 T4096 H16 dk = dv = 128).
 * T = 0 copies dS_final to dS0 and dd_final to dd0 (zeros when NULL).
 * Some per-row sums of a chunk are reduced with shared-memory atomic adds, so
 * two calls on the same inputs can differ in the last bits (the forward
 * entry points are bitwise reproducible).
 * Errors: OSDN_ERR_INVALID_ARG, OSDN_ERR_UNSUPPORTED, OSDN_ERR_CUDA. */
int osdn_bwd_workspace_size(const osdn_params *p, size_t *bytes);

int osdn_bwd(const osdn_params *p,
             const void *q, const void *k, const void *v,
             const void *beta, const void *r,
             const float *d0, const float *S0,
             const void *dout, const float *dS_final, const float *dd_final,
             void *dq, void *dk, void *dv, void *dbeta, void *dr,
             float *dd0, float *dS0,
             void *workspace, size_t workspace_bytes,
             void *cuda_stream);

/* osdn_bwd_gated: the reverse-mode derivative of gated OSDN, the forward that
 * osdn_fwd_gated computes (the recurrence stated above: the OSDN write
 * applied to the decayed state alpha_t S_{t-1}), for the same L as osdn_bwd.
 * Arguments as osdn_bwd,
 * plus alpha [B, T, H] (input dtype, every value in [0, 1]; not NULL when
 * T > 0) and dalpha [B, T, H] (input dtype, overwritten; not NULL when T > 0).
 * Unlike osdn_fwd_gated it takes every dtype and width osdn_bwd takes, plain
 * or anchored APF (the gate does not enter the preconditioner recurrence).
 * Inside a 64-token chunk the gate products run as powers of two of sums of
 * log2 alpha, each term clamped at -120, as in the forward: dalpha is the
 * derivative with respect to alpha_eff = max(alpha, 2^-120), and it stays
 * finite (and accurate) for alpha = 0. The workspace is osdn_bwd's, of
 * osdn_bwd_workspace_size() bytes.
 * Errors: those of osdn_bwd; OSDN_ERR_INVALID_ARG when alpha or dalpha is
 * NULL with T > 0. */
int osdn_bwd_gated(const osdn_params *p,
                   const void *q, const void *k, const void *v,
                   const void *beta, const void *r, const void *alpha,
                   const float *d0, const float *S0,
                   const void *dout, const float *dS_final, const float *dd_final,
                   void *dq, void *dk, void *dv, void *dbeta, void *dr,
                   void *dalpha, float *dd0, float *dS0,
                   void *workspace, size_t workspace_bytes,
                   void *cuda_stream);

/* Largest scratch osdn_fwd_noalloc can use: B * T * H * dk * element size
 * (2 bytes for bf16, 4 for fp32) must not exceed this. */
#define OSDN_NOALLOC_SCRATCH_BYTES (32u << 20)

/* osdn_fwd without a workspace argument, for callers that cannot allocate
 * device memory at call time. Examples: a plugin or extension whose device
 * memory is owned and budgeted by a host framework, or a latency-critical
 * loop that must not enter the CUDA allocator, which can synchronise the
 * device. The pages describe no such variant; the method has no counterpart
 * of it. Arguments and results are those of osdn_fwd.
 *
 * The scaled write keys go to one fixed scratch array inside the library
 * (OSDN_NOALLOC_SCRATCH_BYTES of device memory that every GPU which loads the
 * library keeps until the process exits). The library calls no cudaMalloc or
 * cudaFree for it. Each call made outside stream capture looks up the array's
 * device address (cudaGetSymbolAddress) with the calling device current, so a
 * device reset between calls is harmless; a call made while cuda_stream is
 * capturing reuses the address of that device's last uncaptured call, so make
 * the first call on a device before any stream capture (a captured first call
 * returns OSDN_ERR_INVALID_ARG). Every call uses the same array, and the
 * scan overwrites every scratch entry the chunk phase reads, so stale contents
 * from an earlier call are never used. Two calls that overlap on the GPU (for
 * example on two streams) race on the array: order them on one stream.
 * It never splits sequences into segments (osdn_fwd_segments): where
 * osdn_fwd splits, the two agree up to rounding; elsewhere bit for bit.
 * Errors: those of osdn_fwd; OSDN_ERR_INVALID_ARG when the scratch needed
 * exceeds OSDN_NOALLOC_SCRATCH_BYTES; OSDN_ERR_CUDA when the address lookup
 * fails. */
int osdn_fwd_noalloc(const osdn_params *p,
                     const void *q, const void *k, const void *v,
                     const void *beta, const void *r,
                     const float *d0, const float *S0,
                     void *out, float *final_S, float *final_d,
                     void *cuda_stream);

/* osdn_fwd on HOST buffers, with the transfers pipelined against the compute.
 * q, k, v, beta, r (nullable), d0, S0 (nullable) and out, final_S, final_d
 * (nullable) are dense host tensors in the layouts of osdn_fwd; page-locked
 * memory (cudaHostAlloc, cudaHostRegister) lets the copies run asynchronously and
 * overlap, pageable memory works but serialises them. device_buffer is
 * caller-owned device memory of at least osdn_fwd_host_buffer_size() bytes
 * (16-byte aligned): it holds the whole problem's device copies and one
 * workspace. The B sequences are cut into `groups` groups of consecutive
 * sequences (0: min(B, 8); at most 16). A library-owned non-blocking stream
 * copies each group's inputs in; cuda_stream runs osdn_fwd on the group once
 * they are in; a second library-owned stream copies its results back. So the
 * upload of one group, the compute of another and the download of a third
 * overlap (the link is full duplex). The call forks from cuda_stream and joins
 * back to it by events; the host results are complete once cuda_stream has
 * reached the point of the call. Sequences are independent, so the results
 * equal osdn_fwd's on the whole batch up to the rounding of the segment plan
 * a smaller batch may choose (osdn_fwd_segments). Dense tensors only (the
 * strides of osdn_params must be zero or dense).
 * Errors: OSDN_ERR_INVALID_ARG, OSDN_ERR_UNSUPPORTED, OSDN_ERR_CUDA. */
int osdn_fwd_host(const osdn_params *p,
                  const void *q, const void *k, const void *v,
                  const void *beta, const void *r,
                  const float *d0, const float *S0,
                  void *out, float *final_S, float *final_d,
                  void *device_buffer, size_t device_bytes,
                  int groups, void *cuda_stream);

/* Bytes of device_buffer that osdn_fwd_host needs for these parameters and
 * `groups` (as in osdn_fwd_host), written to *bytes.
 * Errors: OSDN_ERR_INVALID_ARG, OSDN_ERR_UNSUPPORTED. */
int osdn_fwd_host_buffer_size(const osdn_params *p, int groups, size_t *bytes);

/* Waits for the work queued on cuda_stream, then reports whether any bounded
 * device-side wait of the library's kernels gave up since the last call
 * (OSDN_ERR_TIMEOUT) and clears that flag. Returns OSDN_OK when none did,
 * OSDN_ERR_CUDA when the stream itself reports an error. This is the only
 * entry point that synchronises the host. */
int osdn_sync_status(void *cuda_stream);

/* Diagnostics: upper bound, in nanoseconds, on any single device-side wait
 * (mbarrier) of kernels launched after this call; 0 restores the default
 * (4 s). A wait that reaches it makes its CTA stop early (after letting its
 * own copies and MMAs in flight finish), and osdn_sync_status() then reports
 * OSDN_ERR_TIMEOUT; the results of that call are undefined. Meant for tests
 * of the failure path; process-wide, not thread-safe against launches. */
void osdn_set_wait_limit_ns(unsigned long long ns);

/* Message describing the calling thread's most recent error ("" if none).
 * The string is owned by the library and valid until the thread's next call. */
const char *osdn_get_last_error(void);

/* OSDN_ABI_VERSION of the loaded library. */
int osdn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* OSDN_H */
