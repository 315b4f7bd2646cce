/*
 * hm.h -- C ABI of the HedgeMamba mixer-scan library (libhm.so), sm_100a.
 *
 * The library computes the HedgeMamba mixer's causal, normalised, decayed
 * linear-attention scan and the pieces around it:
 *
 *   Hedgehog feature map   phi(x) = softmax([W x + b, -(W x + b)])   over 2p features
 *   decay                  a_t = exp(-softplus(dt_t) * exp(A_log_h))  per (token, head)
 *   recurrence             S_t = a_t S_{t-1} + phi(k_t) v_t^T
 *                          z_t = a_t z_{t-1} + phi(k_t)
 *                          o_t = (phi(q_t)^T S_t) / (phi(q_t)^T z_t)
 *
 * Sources:
 *   "HedgeMamba: fusing linear attention and state space models" (gsyq.cn
 *   news 1418924): sec. 2.1 (Hedgehog map: one Linear layer, concatenation
 *   with its negation, softmax over the feature axis), sec. 2.3 and sec. 5.2
 *   (mixer: value projection, two Hedgehog instances for q and k, the doubled
 *   state giving numerator and denominator, division, gate, out projection;
 *   short conv kept), sec. 5.3 (feature-map listing walk-through).
 *   "Linear attention explained" (cnblogs ying-chease 22790249): sec. 2
 *   (kernel form and associativity), sec. 3 (recurrent form S_i = S_{i-1} +
 *   phi(k_i) v_i^T), sec. 5 (chunkwise mode for prefill, recurrent mode for
 *   decode), the Q/K/V/S shape section ([b, h, n, d], S is d x d_v).
 *   "State space models: Mamba, S4" (quant67 56-ssm): sec. 3.2 (dt through
 *   softplus), sec. 4.2 (associative affine-map composition, used for the
 *   state carry between sequence segments), sec. 6 (chunked SSD algorithm:
 *   matmuls inside a block, recurrence between blocks).
 *
 * Conventions shared by every entry point
 *   Layout    row-major.  Activations are token-major: [B, L, H, X] (X = d,
 *             F = 2p or dv), i.e. element (b, t, h, x) at ((b*L + t)*H + h)*X + x.
 *             States: S [B, H, F, dv] (row = feature f, column = value c),
 *             z [B, H, F].  dt [B, L, H].  A_log [H].  All state is fp32.
 *             Feature order: f < p is the "+" half (exp(u_f)), f >= p the "-" half.
 *   Dtypes    hm_dtype per argument; dt, A_log, biases and states are fp32.
 *   Pointers  device pointers (cudaMalloc'd or equivalent) unless stated.
 *             Every base pointer must be 16-byte aligned.
 *   Ownership the caller owns every buffer.  The library never allocates
 *             or frees device memory and never synchronises the stream
 *             (except hm_get_device_error, which says so).  All work is
 *             enqueued on `stream` in order.
 *   Errors    argument errors are detected on the host before anything is
 *             enqueued and return HM_ERR_INVALID_ARG (or HM_ERR_UNSUPPORTED
 *             for a valid shape that has no kernel); nothing is written.
 *             Launch failures return HM_ERR_CUDA.  A kernel that detects an
 *             internal fault (a bounded wait that expired) records it in a
 *             per-device error word and exits early; hm_get_device_error
 *             reads and clears it.  hm_last_error_detail() gives a
 *             human-readable reason for the last non-OK status on the
 *             calling host thread.  There is no CPU fallback: every result is
 *             produced by this library's own CUDA kernels.
 */
#ifndef HM_H_
#define HM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HM_API __attribute__((visibility("default")))
#else
#define HM_API
#endif

typedef struct CUstream_st *hm_stream_t; /* identical to cudaStream_t */

typedef enum {
    HM_OK = 0,
    HM_ERR_INVALID_ARG = 1,  /* bad pointer, shape, stride or alignment */
    HM_ERR_UNSUPPORTED = 2,  /* valid arguments, but no kernel for this shape/dtype */
    HM_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    HM_ERR_TIMEOUT = 4,      /* a kernel's bounded wait expired (device error word) */
    HM_ERR_DEVICE = 5        /* a kernel reported another internal fault */
} hm_status;

typedef enum { HM_F32 = 0, HM_BF16 = 1 } hm_dtype;

/*
 * Variant flags of the scan and the decode step (the `flags` field of
 * hm_scan_args / hm_decode_args; 0 = the plain recurrence above).
 *
 * HM_FLAG_DT_SCALED_INPUT  the input term is multiplied by the step size
 *     Delta_t = softplus(dt_t), as in Mamba's discretised input B-bar = Delta B
 *     (HedgeMamba explainer sec. 5.2: the mixer calls Mamba's selective scan;
 *     SSM article sec. 3.2):
 *         S_t = a_t S_{t-1} + Delta_t phi(k_t) v_t^T,  z_t = a_t z_{t-1} + Delta_t phi(k_t)
 *     Requires dt.
 * HM_FLAG_PER_FEATURE_DECAY  one decay rate per (head, feature): A_log is
 *     [H, F] and a_{t,f} = exp(-softplus(dt_t) * exp(A_log[h, f])) scales row
 *     f of S and entry f of z (gated linear attention's diag(alpha) S,
 *     linear-attention tutorial sec. 4.4; Mamba-1's A per state dimension).
 *     Requires dt.  Runs on the CUDA-core scan (no tensor-core kernel).
 * HM_FLAG_ROPE  rotary position embedding on phi(q_t) and phi(k_t) before the
 *     recurrence (HedgeMamba explainer sec. 5.2: RoPE on phi(Q), phi(K)), with
 *     the "rotate half" pairing of feature i with feature i + F/2 and angle
 *     pos_t * rope_base^(-2i/F); pos_t = pos0 + t in a scan, positions[b] in a
 *     decode step.  Rotated features may be negative, so the denominator is
 *     no longer positive by construction; no guard is applied (o = num / den).
 */
typedef enum {
    HM_FLAG_DT_SCALED_INPUT = 1u,
    HM_FLAG_PER_FEATURE_DECAY = 2u,
    HM_FLAG_ROPE = 4u
} hm_flag;

/* Static description of a status code.  Never NULL. */
HM_API const char *hm_status_string(hm_status s);

/* Reason for the last non-OK status returned on this host thread ("" if none). */
HM_API const char *hm_last_error_detail(void);

/* Library version string. */
HM_API const char *hm_version(void);

/*
 * hm_featmap -- Hedgehog feature map (HedgeMamba explainer sec. 2.1, 5.3).
 *
 *   u = W_h x_r + b_h          (W_h is [p, d], b_h is [p] or absent)
 *   phi_r = softmax([u, -u])   over the 2p features, "+" half first
 *
 * x      [rows, d] of x_dtype; row r belongs to head h = r mod H (so a
 *        token-major [B, L, H, d] tensor is passed as rows = B*L*H).
 * W      [p, d] of x_dtype for head 0; head h's matrix starts at
 *        W + h * w_head_stride elements (w_head_stride = 0: shared by all heads).
 * bias   fp32 [p] (+ h * p per head when w_head_stride != 0), or NULL.
 * phi    [rows, 2p] of phi_dtype (written).
 * Supported: d and p multiples of 16, 16 <= p <= 256, d <= 512.
 */
HM_API hm_status hm_featmap(const void *x, hm_dtype x_dtype, int64_t rows, int H, int d, int p,
                     const void *W, int64_t w_head_stride, const float *bias,
                     void *phi, hm_dtype phi_dtype, hm_stream_t stream);

/*
 * hm_scan_chunked_fwd -- prefill: feature maps on q and k, then the decayed
 * normalised recurrence over the whole sequence (spec definition;
 * HedgeMamba explainer sec. 2.3 and 5.2; linear-attention tutorial sec. 3 and
 * sec. 5, chunkwise mode).  Computed chunkwise: inside a chunk by dense
 * matmuls with the decay applied elementwise to the masked score tile,
 * between chunks by carrying (S, z); long sequences are split into segments
 * whose states are combined by the associative affine-map composition
 * (SSM article sec. 4.2).  These are exact rewrites of the recurrence.
 */
typedef struct {
    int64_t B, L;          /* batch, sequence length (L >= 0; L = 0 writes only the states) */
    int H;                 /* heads */
    int d;                 /* q/k head dim (input of the Hedgehog projection) */
    int p;                 /* Hedgehog projection width; F = 2p.  Ignored when W_q == NULL */
    int dv;                /* value head dim */
    hm_dtype io_dtype;     /* dtype of q, k, v, W_q, W_k and o */
    const void *q;         /* [B, L, H, d] */
    const void *k;         /* [B, L, H, d] */
    const void *v;         /* [B, L, H, dv] */
    const void *W_q;       /* [p, d] (per head: + h*w_head_stride), or NULL: q, k already
                              are feature vectors (F = d, entries must be > 0) */
    const void *W_k;       /* [p, d] like W_q; must be NULL iff W_q is NULL */
    int64_t w_head_stride; /* elements between heads' W (0 = shared) */
    const float *b_q;      /* [p] bias of the q map (per head like W) or NULL */
    const float *b_k;      /* [p] bias of the k map or NULL */
    const float *dt;       /* [B, L, H] fp32, or NULL: a_t = 1 (no decay) */
    const float *A_log;    /* [H] fp32 ([H, F] with HM_FLAG_PER_FEATURE_DECAY); required with dt */
    const float *S0;       /* [B, H, F, dv] initial state, or NULL (zero) */
    const float *z0;       /* [B, H, F] initial state, or NULL (zero); NULL iff S0 NULL */
    void *o;               /* [B, L, H, dv] of io_dtype (written), or NULL for a state-only
                              call (S_out required): only the final state is computed */
    float *S_out;          /* [B, H, F, dv] final state, or NULL; may alias S0 */
    float *z_out;          /* [B, H, F] final state, or NULL; may alias z0 */
    void *workspace;       /* device scratch of >= hm_scan_workspace_size() bytes, 256-B aligned */
    size_t workspace_bytes;
    unsigned int flags;    /* hm_flag bits (0: the plain recurrence); unknown bits are rejected */
    float *log_decay_out;  /* [B, H] (per-feature decay: [B, H, F]) sum over the call's tokens of
                              log a_t, i.e. the log of the decay the whole call applies to the
                              state it starts from; or NULL.  With S_out of a zero-start call
                              it is the call's affine map S -> exp(.) S + S_out (hm_scan_combine). */
    double rope_base;      /* HM_FLAG_ROPE: base of the rotation angles (> 0, e.g. 10000) */
    int64_t pos0;          /* HM_FLAG_ROPE: position of token 0 of this call (>= 0) */
} hm_scan_args;

/* Bytes of workspace hm_scan_chunked_fwd needs for these arguments (0 on
 * invalid arguments).  Linear in B*L*H (never quadratic in L). */
HM_API size_t hm_scan_workspace_size(const hm_scan_args *a);

HM_API hm_status hm_scan_chunked_fwd(const hm_scan_args *a, hm_stream_t stream);

/*
 * hm_scan_combine -- start states of consecutive sequence segments from their
 * own zero-start results (SSM article sec. 4.2: the maps S -> A S + b compose
 * associatively, (A2, b2) o (A1, b1) = (A2 A1, A2 b1 + b2); here A is the
 * diagonal decay exp(log_decay) and b the segment's zero-start end state).
 *
 * A sequence cut into n_parts consecutive segments (for example one per GPU)
 * is scanned segment by segment with S0 = NULL, S_out, z_out and log_decay_out
 * (o may be NULL).  Part r's results sit in one flat fp32 record at
 * parts + r * part_len, laid out [log_decay | S | z]:
 *     log_decay  BH values (BH * F with per_feature), padded with unread
 *                values to a multiple of 4
 *     S          BH * F * dv values ([BH][F][dv])
 *     z          BH * F values
 * (part_len >= their total; the layout an all-gather of per-rank records
 * produces).  The start state of part r is then
 *     start_0 = (S0, z0) or zero,   start_{r+1} = exp(log_decay_r) (.) start_r + (S_r, z_r)
 * and the segment's outputs are those of a scan with S0 = start_r.
 * only_part = -1 writes every part's start to S_start [n_parts][BH][F][dv] and
 * z_start [n_parts][BH][F]; only_part = r writes just part r's start (one
 * [BH][F][dv] / [BH][F] block).  S_end / z_end (nullable) receive start_{n_parts},
 * the state after the whole sequence.  All pointers device, fp32, 16-byte
 * aligned; part_len a multiple of 4.
 */
typedef struct {
    int64_t n_parts;       /* segments, in sequence order */
    int64_t BH;            /* batch x heads */
    int F, dv;             /* state shape per head */
    int per_feature;       /* log_decay has F values per head (HM_FLAG_PER_FEATURE_DECAY) */
    const float *parts;    /* n_parts records of part_len floats */
    int64_t part_len;
    const float *S0, *z0;  /* start of part 0 ([BH][F][dv], [BH][F]) or NULL (zero) */
    int64_t only_part;     /* -1: all parts' starts; else the one part whose start is written */
    float *S_start, *z_start;
    float *S_end, *z_end;  /* nullable */
} hm_combine_args;

HM_API hm_status hm_scan_combine(const hm_combine_args *a, hm_stream_t stream);

/*
 * hm_scan_bwd -- gradients of a prefill (HedgeMamba explainer sec. 3: the
 * mixer is trained by distillation; SSM article sec. 4.3: the scan's states
 * are recomputed in the backward pass, not stored).  For the loss
 * sum over (b, t, h, c) of dout * o with o = hm_scan_chunked_fwd(...) (plain
 * recurrence, no variant flags, shared Hedgehog weights without bias), it
 * writes the gradients with respect to q, k, v, W_q, W_k, dt, A_log and,
 * when asked, the initial state.  All gradients are fp32.  With W_q == NULL
 * (q, k are the features, F = d), grad_q and grad_k are the gradients of the
 * features and grad_W_q, grad_W_k are not written.  With no tokens
 * (B * L * H == 0) every given gradient of W_q, W_k, A_log and of the initial
 * state is zero (grad_A_log is zeroed when A_log is given, even with dt NULL,
 * since an empty dt tensor may come as NULL).
 * The recurrences run on CUDA cores in fp32, on fp32 features recomputed
 * from q, k; the feature map's gradient products dx = du W and (bf16
 * inputs, p = 128, d a multiple of 64 up to 256) dW = du^T x run on the
 * tensor cores over du split into bf16 hi and lo parts (and W's own
 * remainder for fp32 weights), which carries du to about 2^-17 of itself.
 */
typedef struct {
    int64_t B, L;
    int H, d, p, dv;       /* as in hm_scan_args */
    hm_dtype io_dtype;     /* dtype of q, k, v, W_q, W_k and dout */
    const void *q, *k, *v; /* the forward inputs */
    const void *W_q, *W_k; /* [p, d] shared by all heads, or NULL */
    const float *dt, *A_log; /* as in hm_scan_args (dt NULL: a = 1) */
    const float *S0, *z0;  /* the forward's initial state or NULL */
    const void *dout;      /* [B, L, H, dv] gradient of the loss with respect to o */
    float *grad_q, *grad_k;     /* [B, L, H, d] */
    float *grad_v;              /* [B, L, H, dv] */
    float *grad_W_q, *grad_W_k; /* [p, d] (W_q != NULL) */
    float *grad_dt;             /* [B, L, H] (dt != NULL) */
    float *grad_A_log;          /* [H] (dt != NULL) */
    float *grad_S0, *grad_z0;   /* [B, H, F, dv], [B, H, F], or NULL */
    void *workspace;       /* >= hm_scan_bwd_workspace_size() bytes, 256-B aligned */
    size_t workspace_bytes;
} hm_scan_bwd_args;

HM_API size_t hm_scan_bwd_workspace_size(const hm_scan_bwd_args *a);

HM_API hm_status hm_scan_bwd(const hm_scan_bwd_args *a, hm_stream_t stream);

/*
 * hm_step_decode -- one recurrent step per (batch, head) (linear-attention
 * tutorial sec. 3 and sec. 5, recurrent mode): feature maps on the new q and
 * k, then S <- a S + phi(k) v^T, z <- a z + phi(k), o = phi(q)^T S / phi(q)^T z.
 * S and z are updated in place.
 */
typedef struct {
    int64_t B;             /* independent sequences */
    int H, d, p, dv;       /* as in hm_scan_args; F = 2p (or d when W_q == NULL) */
    hm_dtype io_dtype;     /* dtype of q, k, v, W_q, W_k, o */
    const void *q;         /* [B, H, d] */
    const void *k;         /* [B, H, d] */
    const void *v;         /* [B, H, dv] */
    const void *W_q, *W_k; /* as in hm_scan_args (NULL: q, k are feature vectors) */
    int64_t w_head_stride;
    const float *b_q, *b_k;
    const float *dt;       /* [B, H] fp32 or NULL (a = 1) */
    const float *A_log;    /* [H] fp32 ([H, F] with HM_FLAG_PER_FEATURE_DECAY) */
    float *S;              /* [B, H, F, dv] fp32, read and written */
    float *z;              /* [B, H, F] fp32, read and written */
    void *o;               /* [B, H, dv] of io_dtype (written) */
    void *workspace;       /* >= hm_decode_workspace_size() bytes, 256-B aligned */
    size_t workspace_bytes;
    unsigned int flags;    /* hm_flag bits, as in hm_scan_args */
    double rope_base;      /* HM_FLAG_ROPE: base of the rotation angles (> 0) */
    const int64_t *positions; /* HM_FLAG_ROPE: [B] device int64, position of each sequence's token */
} hm_decode_args;

HM_API size_t hm_decode_workspace_size(const hm_decode_args *a);

HM_API hm_status hm_step_decode(const hm_decode_args *a, hm_stream_t stream);

/*
 * hm_mixer_fwd -- HedgeMamba mixer forward (HedgeMamba explainer sec. 2.3,
 * 5.2; conv and gate kept, sec. 2.2/2.3; gate after the normalisation):
 *
 *   q, k, v, g = x W_{q,k,v,g}^T ;   dt = x W_dt^T (+ b_dt)
 *   q, k, v    = depthwise causal conv of width K (zero left padding) + conv_b
 *   o          = hm_scan_chunked_fwd(q, k, v) per head (d = E/H, Hedgehog W_hq/W_hk)
 *   out        = (o * SiLU(g + b_g)) W_o^T
 *
 * No activation after the conv; no D skip; no RoPE (not part of this path).
 * All matrices bf16 (fp32 accumulation); intermediates are stored in bf16.
 */
typedef struct {
    int64_t B, L;
    int d_model;           /* D */
    int H;                 /* heads; E = H * d_head with d_head = E / H */
    int E;                 /* width of q/k/v/g (= H * d_head) */
    int p;                 /* Hedgehog width (F = 2p) */
    int conv_k;            /* conv width K (1..8) */
    const void *x;         /* [B, L, D] bf16 */
    const void *W_q, *W_k, *W_v, *W_g; /* [E, D] bf16 */
    const void *W_dt;      /* [H, D] bf16 */
    const float *b_dt;     /* [H] or NULL */
    const float *b_g;      /* [E] or NULL */
    const float *conv_w;   /* [3, E, K] fp32 (q, k, v) */
    const float *conv_b;   /* [3, E] fp32 or NULL */
    const void *W_hq, *W_hk; /* [p, d_head] bf16, shared across heads */
    const float *A_log;    /* [H] */
    const void *W_o;       /* [D, E] bf16 */
    void *out;             /* [B, L, D] bf16 (written) */
} hm_mixer_args;

HM_API size_t hm_mixer_workspace_size(const hm_mixer_args *a);

HM_API hm_status hm_mixer_fwd(const hm_mixer_args *a, void *workspace, size_t workspace_bytes,
                       hm_stream_t stream);

/*
 * hm_block_fwd -- the parallel GPT-NeoX / Pythia block with the HedgeMamba
 * mixer in place of attention (HedgeMamba explainer sec. 5.1, Lst. 1: both
 * branches read the block's input through their own norm and add into the
 * residual):
 *
 *   h1  = LN(x; ln1_w, ln1_b),  h2 = LN(x; ln2_w, ln2_b)
 *         LN(x; w, b) = (x - mean) / sqrt(var + eps) * w + b per row of D,
 *         var the population variance
 *   out = x + mixer(h1) + GELU(h2 W_fc1^T + b_fc1) W_fc2^T + b_fc2
 *         GELU(u) = u * Phi(u), the exact (erf) form
 *
 * mixer: the hm_mixer_fwd arguments; its x is the block's input [B, L, D] and
 * its out the block's output [B, L, D] (bf16).  ln*_w, ln*_b: [D] fp32 or NULL
 * (1 and 0).  W_fc1 [d_ff, D], W_fc2 [D, d_ff] bf16; b_fc1 [d_ff], b_fc2 [D]
 * fp32 or NULL.  d_ff a multiple of 64; D a multiple of 256, at most 4096.
 * The caller owns every buffer; workspace (hm_block_workspace_size bytes,
 * 256-byte aligned) holds h1, h2, the fp32 sum x + mixer(h1), the MLP's hidden
 * activations and the mixer's workspace.  Errors: HM_ERR_INVALID_ARG for a
 * null or misaligned pointer, a bad size or a small workspace (nothing is
 * launched); HM_ERR_UNSUPPORTED for sizes the tensor-core GEMM does not take;
 * HM_ERR_CUDA for a launch failure.
 */
typedef struct {
    hm_mixer_args mixer;
    const float *ln1_w, *ln1_b;   /* [D] fp32 or NULL */
    const float *ln2_w, *ln2_b;   /* [D] fp32 or NULL */
    float eps;                    /* > 0 (1e-5 in Pythia) */
    int d_ff;                     /* MLP width (4 D in Pythia) */
    const void *W_fc1;            /* [d_ff, D] bf16 */
    const float *b_fc1;           /* [d_ff] fp32 or NULL */
    const void *W_fc2;            /* [D, d_ff] bf16 */
    const float *b_fc2;           /* [D] fp32 or NULL */
} hm_block_args;

HM_API size_t hm_block_workspace_size(const hm_block_args *a);

HM_API hm_status hm_block_fwd(const hm_block_args *a, void *workspace, size_t workspace_bytes,
                       hm_stream_t stream);

/*
 * hm_step_decode_noalloc -- hm_step_decode for callers that cannot allocate
 * device memory (for example a plugin whose host application owns all device
 * memory and offers no allocator, or a serving loop that must not allocate
 * after start-up).  There is no counterpart in the paper; it is a deployment
 * convenience.  Same arguments, checks and results (bit-identical) as
 * hm_step_decode, except that workspace / workspace_bytes are ignored: the
 * fp32 feature vectors live in a fixed device array inside the library (two
 * planes of 524,288 fp32 values, 4 MiB, held by every GPU that loads the
 * library until the process exits).
 * Limit: when W_q != NULL, B * H * F must not exceed 524,288; larger calls
 * return HM_ERR_INVALID_ARG before anything is enqueued (use hm_step_decode).
 * All calls share that array, so calls whose kernels may overlap on a GPU
 * (several streams or host threads on one device) race and must be serialised
 * by the caller.  The first call on each device looks up the array's device
 * address and caches it for the process; make that first call before any
 * stream capture, and do not call this entry point after cudaDeviceReset.
 */
HM_API hm_status hm_step_decode_noalloc(const hm_decode_args *a, hm_stream_t stream);

/* Number of kernels this library has enqueued in this process so far (all
 * devices, all threads).  A diagnostic for launch accounting. */
HM_API uint64_t hm_launch_count(void);

/* Synchronises `stream`, then returns and clears the calling device's error
 * word: HM_OK, HM_ERR_TIMEOUT (a bounded wait expired) or HM_ERR_DEVICE. */
HM_API hm_status hm_get_device_error(hm_stream_t stream);

/* Diagnostic with no counterpart in the method: enqueues one thread block on
 * `stream` that waits on a barrier nothing ever signals, polling it at most
 * `polls` times (1 .. 2^20) with the same bounded wait the library's
 * pipelined kernels use, then records HM_ERR_TIMEOUT in the device error
 * word, as a stalled pipeline would.  Returns HM_OK once enqueued,
 * HM_ERR_INVALID_ARG for a bad poll count.  Read the recorded status with
 * hm_get_device_error; the context remains usable afterwards. */
HM_API hm_status hm_selftest_wait_timeout(uint32_t polls, hm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HM_H_ */
