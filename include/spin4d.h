/*
 * spin4d.h -- C ABI of the B200-native SPIN-4DGS per-Gaussian attribute decoder.
 *
 * What the library computes (from "Implicit 4D Gaussian Splatting for Fast
 * Motion with Large Inter-Frame Displacements", SPIN-4DGS, sections 3.1 and
 * 3.3): each spatiotemporal Gaussian position (x, y, z, t) is normalised
 * (Eq. 7 scene contraction, Eq. 8 time normalisation), encoded by a 4D
 * multiresolution hash grid (Eq. 9), decoded by a shared trunk and a
 * multibranch head (Eq. 10) into scale, rotation, colour and opacity with the
 * activations of Eq. 11, and turned into a covariance Sigma = R S S^T R^T
 * (Eq. 2).  The backward pass scatter-adds gradients into the hash tables and
 * the network weights; Adam (section 4, implementation details) updates them.
 * A HexPlane encoder with a two-branch deformation network (4D Gaussian
 * Splatting reading notes, sections 3.1-3.2) is a second encoder behind the
 * same covariance assembly, and a double-sigmoid temporal window (KineticGS
 * notes, "learnable energy-flow activation") can gate the opacity.
 *
 * Conventions shared by every call:
 *  - All array pointers are DEVICE pointers owned by the caller unless a
 *    comment says otherwise.  The library never frees or keeps them.
 *  - Every compute call is asynchronous on `stream` (NULL = the legacy
 *    default stream), allocates no memory and never synchronises.
 *  - Arguments are validated on the host before any launch; on a validation
 *    failure nothing is launched and SPIN4D_ERR_INVALID (or
 *    SPIN4D_ERR_UNSUPPORTED for a valid but unimplemented shape) is returned.
 *    A launch failure returns SPIN4D_ERR_CUDA; spin4d_last_cuda_error() gives
 *    the cudaError_t value.
 *  - Gradient outputs ACCUMULATE (+=): the caller zeroes them first.  This is
 *    what lets many batches add into one gradient before one Adam step.
 *  - Arrays are row-major; "N x k" means N rows of k contiguous values.
 *  - Environment variable SPIN4D_FAULT=<name> (for example
 *    SPIN4D_FAULT=spin4d_decode_fwd) makes that entry point return
 *    SPIN4D_ERR_INJECTED after validation and before any launch; it exists
 *    to test callers' error paths without touching the GPU.
 */
#ifndef SPIN4D_H
#define SPIN4D_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA include. */
typedef struct CUstream_st* spin4d_stream_t;

typedef enum spin4d_status {
    SPIN4D_OK = 0,
    SPIN4D_ERR_INVALID = -1,      /* bad argument; nothing launched */
    SPIN4D_ERR_UNSUPPORTED = -2,  /* valid but not implemented shape; nothing launched */
    SPIN4D_ERR_CUDA = -3,         /* a CUDA launch or query failed */
    SPIN4D_ERR_NONFINITE = -4,    /* a kernel met a non-finite value (see spin4d_adam_step) */
    SPIN4D_ERR_INJECTED = -5,     /* SPIN4D_FAULT selected this call */
    SPIN4D_ERR_TIMEOUT = -6,      /* a kernel's bounded wait ran out (see spin4d_check_device_errors) */
    SPIN4D_ERR_BOUNDS = -7        /* checked build: a device bounds check failed */
} spin4d_status;

typedef enum spin4d_dtype { SPIN4D_F32 = 0, SPIN4D_F16 = 1 } spin4d_dtype;

#define SPIN4D_MAX_LEVELS 16
#define SPIN4D_MAX_FEATURES 8
#define SPIN4D_MAX_WIDTH 128

/* grid flag: `pos` already holds x~ in [0,1]^4; skip Eq. 7-8 (values are clamped to [0,1]). */
#define SPIN4D_INPUT_NORMALISED 1u

/*
 * 4D multiresolution hash grid (SPIN-4DGS section 3.3, Eq. 9).
 * Level l owns T = 2^log2_T entries of F features; table memory is
 * L x T x F values of `table_dtype`, entry-major (the F features of an entry
 * are contiguous), level after level.  res[l][d] is the number of grid
 * VERTICES along axis d (x, y, z, t) at level l (>= 2), so a normalised
 * coordinate u in [0,1] sits at u * (res - 1).  A level whose vertex count
 * res_x*res_y*res_z*res_t is <= T is indexed densely (x fastest); otherwise by
 * the spatial hash (v_x*1 ^ v_y*2654435761 ^ v_z*805459861 ^ v_t*3674653429)
 * mod 2^32, mod T.  Time is normalised by (t - t_min)/(t_max - t_min)
 * (Eq. 8) and clamped to [0,1].
 */
typedef struct spin4d_grid_desc {
    int32_t L;              /* levels, 1..16 */
    int32_t F;              /* features per level: 1, 2, 4 or 8 */
    int32_t log2_T;         /* entries per level = 2^log2_T, 4..24 */
    int32_t table_dtype;    /* spin4d_dtype of the tables */
    int32_t res[SPIN4D_MAX_LEVELS][4];
    float t_min, t_max;     /* t_max > t_min */
    uint32_t flags;         /* SPIN4D_INPUT_NORMALISED or 0 */
    int32_t reserved;       /* must be 0 */
} spin4d_grid_desc;

/*
 * Fills `g`.  Per-level resolutions follow Instant-NGP's geometric growth,
 * res_l = floor(Nmin * b^l) with b = exp((ln Nmax - ln Nmin)/(L - 1)),
 * separately for the spatial axes (nmin_s..nmax_s) and time (nmin_t..nmax_t).
 * Host only; returns SPIN4D_ERR_INVALID on bad sizes.
 */
int spin4d_grid_init(spin4d_grid_desc* g, int L, int F, int log2_T, int table_dtype,
                     int nmin_s, int nmax_s, int nmin_t, int nmax_t,
                     float t_min, float t_max);

/*
 * Decoder network (SPIN-4DGS section 3.3, Eq. 10): a trunk of n_hidden
 * ReLU layers of width `hidden` on the LF-dimensional latent, then one linear
 * layer of 11 rows [scale 3 | rotation 4 | rgb 3 | opacity 1].
 * Weights are ONE packed vector of `w_dtype`: for each layer in order,
 * W[out][in] row-major followed by b[out].  in_dim must equal L*F.
 * gate != 0 multiplies the opacity by the double-sigmoid window
 * sigmoid((t~-(c-r))/tau) * sigmoid(((c+r)-t~)/tau) of the normalised time t~,
 * with per-Gaussian (c, r) passed in `gate_cr`.
 */
typedef struct spin4d_mlp_desc {
    int32_t in_dim;     /* = L*F, <= 128 */
    int32_t hidden;     /* trunk width, 1..128 */
    int32_t n_hidden;   /* trunk layers, 1..4 */
    int32_t w_dtype;    /* spin4d_dtype of the packed weights */
    int32_t gate;       /* 0 or 1 */
    float tau;          /* > 0 when gate != 0 */
} spin4d_mlp_desc;

/* Number of values in the packed weight vector (or -1 if `m` is invalid). */
int64_t spin4d_mlp_param_count(const spin4d_mlp_desc* m);

/* Decoded attributes, structure of arrays, fp32, device memory:
 * scale N x 3, rot N x 4 (unit, (w,x,y,z)), rgb N x 3, opacity N x 1,
 * cov N x 6 packed (xx, xy, xz, yy, yz, zz).  None of these may be NULL.
 * latent (optional, may be NULL): N x (L*F) fp32, 16-byte aligned, receives
 * the encoder output z (Eq. 9) so that a following spin4d_decode_bwd can
 * read it instead of gathering the tables again. */
typedef struct spin4d_outputs {
    float* scale;
    float* rot;
    float* rgb;
    float* opacity;
    float* cov;
    float* latent;
} spin4d_outputs;

/* Upstream gradients on the decoded attributes, same shapes as spin4d_outputs.
 * A NULL member means a zero gradient for that attribute. */
typedef struct spin4d_output_grads {
    const float* scale;
    const float* rot;
    const float* rgb;
    const float* opacity;
    const float* cov;
} spin4d_output_grads;

/*
 * Eq. 7-9: normalise and hash-encode N positions.
 *   pos     N x 4 fp32 (x, y, z, t), 16-byte aligned
 *   tables  L x T x F of g->table_dtype, aligned to F * sizeof(dtype)
 *   z       N x (L*F) fp32 output, level-major (z[n][l*F + f])
 * N == 0 is valid and launches nothing.
 */
int spin4d_encode_fwd(const spin4d_grid_desc* g, const float* pos, int64_t N,
                      const void* tables, float* z, spin4d_stream_t stream);

/*
 * Eq. 7-11 and Eq. 2 fused: normalise, encode, trunk + head, activations
 * s = exp(min(s^, 20)), r = r^/max(||r^||, 1e-12), rgb = sigmoid, o = sigmoid
 * (times the gate when m->gate), then Sigma.  One kernel, nothing but `out`
 * written to memory.
 *   weights  packed vector, see spin4d_mlp_desc, 16-byte aligned
 *   gate_cr  N x 2 fp32 (c, r) when m->gate, else ignored (may be NULL)
 */
int spin4d_decode_fwd(const spin4d_grid_desc* g, const spin4d_mlp_desc* m,
                      const float* pos, int64_t N, const void* tables, const void* weights,
                      const float* gate_cr, spin4d_outputs out, spin4d_stream_t stream);

/* Bytes of device workspace spin4d_decode_bwd needs for N positions. */
size_t spin4d_decode_bwd_workspace(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, int64_t N);

/*
 * Backward of spin4d_decode_fwd for loss = sum_k <grad_out.k, output_k>:
 * recomputes the forward (from `latent`, the z that spin4d_decode_fwd saved
 * for the same positions and tables, when it is not NULL; otherwise by
 * gathering the tables again), then accumulates
 *   grad_tables   += dloss/dtables   (L x T x F fp32, scatter-added with atomics)
 *   grad_weights  += dloss/dweights  (packed like `weights`, fp32)
 * The gradient of s^ is zero where s^ > 20 (the clip); ReLU passes where its
 * input is > 0.  `workspace` (device, >= spin4d_decode_bwd_workspace bytes,
 * 256-byte aligned, contents ignored on entry) holds per-block partial weight
 * gradients so that grad_weights is summed in a fixed order.
 */
int spin4d_decode_bwd(const spin4d_grid_desc* g, const spin4d_mlp_desc* m,
                      const float* pos, int64_t N, const void* tables, const void* weights,
                      const float* gate_cr, const float* latent, const spin4d_output_grads* grad_out,
                      float* grad_tables, float* grad_weights,
                      void* workspace, size_t ws_bytes, spin4d_stream_t stream);

/*
 * Optional extra gradients of spin4d_decode_bwd_ext (a NULL member is not
 * computed).  Both are accumulated (+=) and each position's values are
 * written by one thread (no atomics), so repeated calls add identically.
 *
 * pos (N x 3 fp32, 4-byte aligned): dloss/d(x, y, z) of the Gaussian means
 *   (SPIN-4DGS section 3.3 trains the positions jointly with the decoder),
 *   through the quadrilinear interpolation weights of every level (the
 *   derivative inside the cell the position falls in, times res - 1 per
 *   axis) and the Jacobian of Eq. 7 (I/4 inside the unit ball; outside, the
 *   contracted point 2 - 1/|mu| along the ray of mu).  With
 *   SPIN4D_INPUT_NORMALISED it is the gradient w.r.t. the normalised
 *   coordinates, zero where the clamp to [0, 1] bound.  The timestamp is
 *   data, not a parameter: it gets no gradient.  The corner entries are
 *   gathered again for this even when `latent` is given.
 * gate_cr (N x 2 fp32, 4-byte aligned; gated decoders only): dloss/d(c, r)
 *   of the KineticGS window (a learned gate: c and r come from the caller's
 *   own predictor).  o = sigma(o^) w, w = a b, a = sigma((t - (c - r))/tau),
 *   b = sigma(((c + r) - t)/tau): dloss/dw = g_o sigma(o^), dw/dc =
 *   a b (a - b)/tau, dw/dr = a b (2 - a - b)/tau.
 */
typedef struct spin4d_extra_grads {
    float* pos;
    float* gate_cr;
} spin4d_extra_grads;

/* spin4d_decode_bwd plus the gradients `extra` asks for (extra not NULL;
 * SPIN4D_ERR_INVALID for extra->gate_cr on an ungated decoder).  Other
 * arguments, results and errors are those of spin4d_decode_bwd. */
int spin4d_decode_bwd_ext(const spin4d_grid_desc* g, const spin4d_mlp_desc* m,
                          const float* pos, int64_t N, const void* tables, const void* weights,
                          const float* gate_cr, const float* latent, const spin4d_output_grads* grad_out,
                          float* grad_tables, float* grad_weights, const spin4d_extra_grads* extra,
                          void* workspace, size_t ws_bytes, spin4d_stream_t stream);

/*
 * spin4d_decode_bwd without a workspace argument, for callers that cannot
 * allocate device memory (hosts that own all device memory and hand the
 * library only its input and output buffers, or loops that may not call
 * cudaMalloc while running).  The paper has no counterpart; this is an
 * interface convenience of this library.
 *
 * The scratch lives in one array of SPIN4D_NOALLOC_SCRATCH_BYTES compiled
 * into the library; every GPU that loads the library holds it until the
 * process exits.  Returns SPIN4D_ERR_INVALID, launching nothing, when the
 * scratch this (g, m, N) needs (spin4d_decode_bwd_workspace) is larger.
 * The first call on each device looks the array's device address up
 * (cudaGetSymbolAddress, with that device current) and keeps it for the life
 * of the process; make that first call before any stream capture.  A device
 * reset (cudaDeviceReset, or the primary context destroyed and created again)
 * can move the array, and the kept address is then stale: do not call this
 * entry point after resetting a device it has already run on.  All calls share the one array: calls that
 * overlap on the GPU (different streams, or different host threads) race and
 * corrupt each other's weight gradients; serialise them.  Each call writes
 * every part of the scratch it reads, so nothing needs clearing between calls.
 * Other arguments, results and errors are those of spin4d_decode_bwd.
 */
#define SPIN4D_NOALLOC_SCRATCH_BYTES (16u << 20)
/* The size of that array as this library was compiled (bytes). */
size_t spin4d_decode_bwd_noalloc_scratch_bytes(void);
int spin4d_decode_bwd_noalloc(const spin4d_grid_desc* g, const spin4d_mlp_desc* m,
                              const float* pos, int64_t N, const void* tables, const void* weights,
                              const float* gate_cr, const float* latent, const spin4d_output_grads* grad_out,
                              float* grad_tables, float* grad_weights, spin4d_stream_t stream);

/*
 * Eq. 2 alone: Sigma = R(q) diag(s)^2 R(q)^T for unit quaternions q = (w,x,y,z).
 *   scale N x 3, rot N x 4 (used as given, not renormalised), cov N x 6 packed.
 */
int spin4d_cov_assemble(const float* scale, const float* rot, int64_t N, float* cov,
                        spin4d_stream_t stream);

/*
 * Adam (Kingma & Ba) with bias correction, step counted from 1:
 *   m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2;
 *   p -= lr * (m / (1-b1^step)) / (sqrt(v / (1-b2^step)) + eps)
 * over n fp32 parameters `params` with fp32 state m, v (zero before step 1).
 * params_work (may be NULL) receives an fp16 copy of the updated parameters
 * (the working copy fp16 tables / weights are read from).  zero_grad != 0
 * clears `grad` after use.  If `nonfinite_flag` is non-NULL (device int32,
 * caller-zeroed), it is set to 1 when any updated parameter is not finite;
 * the host reads it when it chooses (the call itself never synchronises).
 */
int spin4d_adam_step(float* params, void* params_work, float* grad, float* m, float* v,
                     int64_t n, int step, float lr, float b1, float b2, float eps,
                     int zero_grad, int32_t* nonfinite_flag, spin4d_stream_t stream);

/*
 * HexPlane encoder + deformation network (4D Gaussian Splatting reading
 * notes, sections 3.1-3.2).  Planes XY, XZ, YZ, XT, YT, ZT at each spatial
 * resolution scales[s] (time axis: time_res samples), `channels` each,
 * stored fp32 channel-last [rows = second axis][cols = first axis][C],
 * scale-major then plane order; sampled bilinearly (align corners) at
 * x~ = (mu + 1)/2 and t~ = frame/(n_frames - 1); samples concatenated
 * (scale, plane, channel) into n_scales*6*channels features; trunk of
 * n_hidden ReLU layers of width `hidden`; one 58-row linear layer
 * [d_mu 3 | d_q 4 | d_logs 3 | d_sh 48]; weights packed fp32 as in
 * spin4d_mlp_desc.
 */
typedef struct spin4d_hexplane_desc {
    int32_t n_scales;       /* 1..4 */
    int32_t scales[4];      /* spatial resolutions (vertices), >= 2 */
    int32_t time_res;       /* time samples, >= 2 */
    int32_t channels;       /* 32 (multiple of 4, <= 32) */
    int32_t n_frames;       /* frames of the sequence, >= 2 */
    int32_t hidden;         /* trunk width, <= 128 */
    int32_t n_hidden;       /* trunk layers, 1..4 */
} spin4d_hexplane_desc;

/* Values in the packed plane array / weight vector (-1 if invalid). */
int64_t spin4d_hexplane_plane_count(const spin4d_hexplane_desc* h);
int64_t spin4d_hexplane_param_count(const spin4d_hexplane_desc* h);

/* Deformed Gaussians: mu' N x 3, rot N x 4, scale N x 3, sh N x 48, cov N x 6 (fp32).
 * latent (optional, may be NULL): N x (n_scales*6*channels) fp32, 32-byte
 * aligned, receives the concatenated plane samples.
 * hidden (optional, may be NULL): N x hidden fp32, 16-byte aligned, receives
 * the first trunk layer's output h1 = relu(W1 z + b1).  Saved beside the
 * latent, it spares the backward the first layer (spin4d_hexplane_bwd_saved). */
typedef struct spin4d_hex_outputs {
    float* mu;
    float* rot;
    float* scale;
    float* sh;
    float* cov;
    float* latent;
    float* hidden;
} spin4d_hex_outputs;

typedef struct spin4d_hex_output_grads {
    const float* mu;
    const float* rot;
    const float* scale;
    const float* sh;
    const float* cov;
} spin4d_hex_output_grads;

/*
 * mu' = mu + d_mu; q' = (q_can + d_q)/max(||q_can + d_q||, 1e-12);
 * s' = exp(logs_can + d_logs); sh' = sh_can + d_sh; Sigma(s', q').
 *   mu N x 3, frame N int32 in [0, n_frames), q_can N x 4, logs_can N x 3,
 *   sh_can N x 48 (all fp32).  planes and weights: device, 32-byte aligned;
 *   out.rot, out.sh and sh_can 16-byte aligned.  Misaligned or NULL arguments return
 *   SPIN4D_ERR_INVALID; channels other than 32, hidden other than 64 or
 *   n_hidden other than 2 return SPIN4D_ERR_UNSUPPORTED, before any launch.
 */
int spin4d_hexplane_fwd(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame,
                        int64_t N, const float* planes, const float* weights,
                        const float* q_can, const float* logs_can, const float* sh_can,
                        spin4d_hex_outputs out, spin4d_stream_t stream);

size_t spin4d_hexplane_bwd_workspace(const spin4d_hexplane_desc* h, int64_t N);

/*
 * Backward of spin4d_hexplane_fwd: grad_planes += dL/dplanes and
 * grad_weights += dL/dweights (fp32, packed like planes and weights) for
 * L = sum over outputs of <grad_out.x, x>; a NULL member of grad_out is a
 * zero gradient.  latent (optional, may be NULL, 32-byte aligned) is the
 * forward's saved latent for the same inputs; given, the plane samples are
 * read from it instead of being gathered again.  workspace: device memory
 * of at least spin4d_hexplane_bwd_workspace(h, N) bytes, 256-byte aligned,
 * owned by the caller, overwritten (per-block weight-gradient partials, and
 * with a saved latent N x 64 fp32 of hidden-layer gradients handed between
 * the two kernels of that path).  Plane gradients are accumulated with
 * fp32 atomics (their order of summation is not fixed); weight gradients
 * are summed in a fixed order.
 */
int spin4d_hexplane_bwd(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame,
                        int64_t N, const float* planes, const float* weights,
                        const float* q_can, const float* logs_can, const float* sh_can,
                        const float* latent, const spin4d_hex_output_grads* grad_out,
                        float* grad_planes, float* grad_weights,
                        void* workspace, size_t ws_bytes, spin4d_stream_t stream);

/*
 * The energy-flow window of the KineticGS notes ("learnable energy-flow
 * activation") on the HexPlane deformation.  Each Gaussian carries a window
 * centre c and half-width r; on the normalised time t~ = frame/(n_frames - 1)
 *   w = sigma((t~ - (c - r))/tau) sigma(((c + r) - t~)/tau).
 * The notes gate the spatial displacement with a binary H(w) in {0, 1}, so a
 * Gaussian moves only inside its window, and modulate the scale and the
 * features continuously by w.  Read here as H(w) = [w >= 1/2] and
 *   mu' = mu + H(w) d_mu,  s' = exp(logs_can + w d_logs),  sh' = sh_can + w d_sh,
 * with the rotation offset (not among the quantities the notes modulate)
 * applied as without the window.  H has zero derivative: c and r receive
 * gradient through w alone.
 *   cr:      N x 2 (c, r) fp32, device, 8-byte aligned.
 *   tau:     > 0 and finite.
 *   grad_cr: backward only: N x 2 fp32, 8-byte aligned, += d loss / d(c, r);
 *            NULL for none.  Each Gaussian's pair is written by one thread.
 */
typedef struct spin4d_hex_gate {
    const float* cr;
    float tau;
    float* grad_cr;
} spin4d_hex_gate;

/* spin4d_hexplane_fwd with the window (gate not NULL).  Other arguments,
 * results and errors are those of spin4d_hexplane_fwd; SPIN4D_ERR_INVALID for
 * a bad gate or a non-NULL gate->grad_cr. */
int spin4d_hexplane_fwd_gated(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame,
                              int64_t N, const float* planes, const float* weights,
                              const float* q_can, const float* logs_can, const float* sh_can,
                              const spin4d_hex_gate* gate, spin4d_hex_outputs out, spin4d_stream_t stream);

/* spin4d_hexplane_bwd with the window (gate not NULL), and d loss / d(c, r)
 * into gate->grad_cr when given.  Other arguments, results and errors are
 * those of spin4d_hexplane_bwd; SPIN4D_ERR_UNSUPPORTED where only the fp32
 * SIMT kernels could run. */
int spin4d_hexplane_bwd_gated(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame,
                              int64_t N, const float* planes, const float* weights,
                              const float* q_can, const float* logs_can, const float* sh_can,
                              const float* latent, const spin4d_hex_gate* gate,
                              const spin4d_hex_output_grads* grad_out,
                              float* grad_planes, float* grad_weights,
                              void* workspace, size_t ws_bytes, spin4d_stream_t stream);

/* The forward's saved activations for spin4d_hexplane_bwd_saved: latent as
 * in spin4d_hex_outputs (required), hidden the matching h1 (NULL: the
 * backward computes h1 again from the latent). */
typedef struct spin4d_hex_saved {
    const float* latent;
    const float* hidden;
} spin4d_hex_saved;

/*
 * spin4d_hexplane_bwd (gate NULL) or spin4d_hexplane_bwd_gated (gate given)
 * from the forward's saved latent and, when saved->hidden is given, its
 * saved h1: the backward then starts at the second layer.  The results and
 * every other argument are those of the two calls.  SPIN4D_ERR_INVALID for
 * a NULL saved or saved->latent, a misaligned saved->hidden (16 bytes) or a
 * bad gate; SPIN4D_ERR_UNSUPPORTED where only the fp32 SIMT kernels could
 * run.  The saved arrays must come from a forward with the same inputs,
 * planes and weights (and window): they are not checked.
 */
int spin4d_hexplane_bwd_saved(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame,
                              int64_t N, const float* planes, const float* weights,
                              const float* q_can, const float* logs_can, const spin4d_hex_saved* saved,
                              const spin4d_hex_gate* gate, const spin4d_hex_output_grads* grad_out,
                              float* grad_planes, float* grad_weights,
                              void* workspace, size_t ws_bytes, spin4d_stream_t stream);

/*
 * Test hook: the interpolation cell of every position at every level, as the
 * kernels compute it.  idx N x L x 16 uint32 (corner c selects vertex
 * base_d + bit d of c, d = 0 x, 1 y, 2 z, 3 t); frac N x L x 4 fp32
 * (position inside the cell, per axis).
 */
int spin4d_debug_corners(const spin4d_grid_desc* g, const float* pos, int64_t N,
                         uint32_t* idx, float* frac, spin4d_stream_t stream);

/*
 * Synchronous: reads the library's device error word, set by a kernel whose
 * bounded wait for its own tensor-core work ran out (the kernel then frees
 * its tensor memory and exits early, leaving its outputs incomplete).
 * Returns SPIN4D_OK or SPIN4D_ERR_TIMEOUT; clear != 0 resets the word.  In
 * the checked build (spin4d_checked_build) also SPIN4D_ERR_BOUNDS when a
 * device bounds check failed (it takes precedence; clear resets those
 * words too).  Waits for the current device's legacy default stream.
 */
int spin4d_check_device_errors(int clear);

/*
 * The paper's attribute-aware decoder (SPIN-4DGS section 3.3, Eqs. 9-11):
 * four heads -- scale, rotation, spherical-harmonic colour, opacity -- each a
 * three-layer MLP in_dim -> hidden -> hidden -> rows (3, 4, sh_dim, 1) with
 * exact GELU (x Phi(x)) after the first two layers, on the shared latent z
 * of the hash encoder; s = exp(min(s^, 20)) (gradient zero above 20),
 * r = r^/max(|r^|, 1e-12), sh = sh^, o = sigma(o^); Sigma by Eq. 2.
 * Weights (fp32 or fp16, 4-byte aligned) are packed head by head in that
 * order, each [W1 b1 W2 b2 W3 b3] with W[out][in] row-major.
 * in_dim = L*F; in_dim, hidden and sh_dim at most 64, in_dim and hidden
 * multiples of 4 (SPIN4D_ERR_UNSUPPORTED otherwise).  fp32 arithmetic, except
 * that the forward with fp16 tables and weights, F = 4, in_dim = hidden = 64,
 * sh_dim = 48 and 16-byte aligned sh and raw runs its layers on the tensor
 * cores: z and the hidden activations are rounded to
 * fp16, products accumulate in fp32 (the latent output stays fp32).
 */
typedef struct spin4d_heads_desc {
    int32_t in_dim;
    int32_t hidden;         /* 64 in the paper */
    int32_t sh_dim;         /* 48: degree-3 SH, three colour channels */
    int32_t w_dtype;        /* SPIN4D_F32 or SPIN4D_F16 */
} spin4d_heads_desc;

/* scale N x 3, rot N x 4 (16-byte aligned), sh N x sh_dim, opacity N x 1,
 * cov N x 6 (fp32); latent (optional) N x in_dim receives z; raw
 * (optional) N x 8 receives the raw outputs of the scale, rotation and
 * opacity heads (s^ 3, r^ 4, o^ 1), which spin4d_heads_bwd can take instead
 * of recomputing those heads. */
typedef struct spin4d_heads_outputs {
    float* scale;
    float* rot;
    float* sh;
    float* opacity;
    float* cov;
    float* latent;
    float* raw;
} spin4d_heads_outputs;

typedef struct spin4d_heads_output_grads {
    const float* scale;
    const float* rot;
    const float* sh;
    const float* opacity;
    const float* cov;
} spin4d_heads_output_grads;

/* Values in the packed weight vector (-1 if invalid). */
int64_t spin4d_heads_param_count(const spin4d_heads_desc* h);

/* Bytes of the forward's optional workspace: N rows of 64 fp16 features for
 * the configuration whose layers run on the tensor cores (see
 * spin4d_heads_desc), 0 for every other configuration. */
size_t spin4d_heads_fwd_workspace(const spin4d_grid_desc* g, const spin4d_heads_desc* h, int64_t N);

/* Forward of the four heads for N positions (device pointers; pos N x 4,
 * tables and weights as above).  workspace (device, 256-byte aligned,
 * >= spin4d_heads_fwd_workspace bytes; may be NULL) lets the tensor-core
 * configuration run as two kernels: a full-occupancy hash gather that writes
 * z (fp16) there, then the layers; with NULL the same arithmetic runs as one
 * fused kernel, slower.  Other configurations ignore it.  Misaligned or too
 * small a workspace returns SPIN4D_ERR_INVALID. */
int spin4d_heads_fwd(const spin4d_grid_desc* g, const spin4d_heads_desc* h, const float* pos, int64_t N,
                     const void* tables, const void* weights, spin4d_heads_outputs out, void* workspace,
                     size_t ws_bytes, spin4d_stream_t stream);

size_t spin4d_heads_bwd_workspace(const spin4d_grid_desc* g, const spin4d_heads_desc* h, int64_t N);

/* Backward of spin4d_heads_fwd for loss = sum_k <grad_out.k, output_k>
 * (NULL members are zero): grad_tables += (L x T x F fp32, atomics),
 * grad_weights += (packed like weights, fp32, summed in a fixed order).
 * latent and raw (optional, each may be NULL) are the z and the raw head
 * outputs spin4d_heads_fwd saved for the same inputs; workspace as for
 * spin4d_decode_bwd, >= spin4d_heads_bwd_workspace bytes.  With both given
 * (latent 16-byte aligned) the tensor-core configuration of spin4d_heads_desc
 * runs its layers on the tensor cores with fp16 operands (z, activations,
 * output adjoints, deltas) and fp32 accumulation; otherwise fp32 SIMT. */
int spin4d_heads_bwd(const spin4d_grid_desc* g, const spin4d_heads_desc* h, const float* pos, int64_t N,
                     const void* tables, const void* weights, const float* latent, const float* raw,
                     const spin4d_heads_output_grads* grad_out, float* grad_tables, float* grad_weights,
                     void* workspace, size_t ws_bytes, spin4d_stream_t stream);

/*
 * Adam with per-group learning rates (SPIN-4DGS section 4 uses separate
 * rates for the encoder and each decoder head): spin4d_adam_step over
 * params[0..n) where element i takes the learning rate of the first group
 * whose `end` exceeds i (groups sorted by end, the last end = n, at most
 * SPIN4D_MAX_ADAM_GROUPS; host array).  Other arguments as spin4d_adam_step.
 */
#define SPIN4D_MAX_ADAM_GROUPS 16
typedef struct spin4d_adam_group {
    int64_t end;
    float lr;
} spin4d_adam_group;
int spin4d_adam_step_groups(float* params, void* params_work, float* grad, float* m, float* v, int64_t n,
                            const spin4d_adam_group* groups, int n_groups, int step, float b1, float b2, float eps,
                            int zero_grad, int32_t* nonfinite_flag, spin4d_stream_t stream);

/* Learning rate at optimiser step `step` (from 1): linear warm-up from 0 to
 * lr_max over `warmup` steps, then cosine decay to lr_min at step `total`
 * (lr_min afterwards).  Host function. */
double spin4d_lr_warmup_cosine(int64_t step, double lr_max, double lr_min, int64_t warmup, int64_t total);

/*
 * Z-order (Morton) ordering of the Gaussians, for gather locality (the
 * KineticGS notes serialise particles onto a Z-order space-filling curve to
 * keep spatial neighbours adjacent).  Decoding the Gaussians in this order
 * makes each tile's positions neighbours, so their hash-table corners
 * overlap in the caches.
 *
 * keys[n]: the 30-bit Z-order code of Gaussian n's normalised spatial
 * coordinates (Eq. 7, the same fp32 arithmetic and SPIN4D_INPUT_NORMALISED
 * handling as the decoder), 10 bits per axis, q = min(floor(mu_bar * 1024),
 * 1023), bit b of axis d at bit 3b + d.  The time coordinate is not used.
 * On return `keys` holds the codes sorted ascending and perm[i] is the input
 * index of the i-th smallest, equal codes in input order (a stable sort: the
 * result is deterministic).  pos N x 4 fp32 (16-byte aligned), keys and perm
 * N uint32 (device, 4-byte aligned), workspace >=
 * spin4d_morton_order_workspace(N) bytes (device, 256-byte aligned).
 * 0 <= N <= SPIN4D_MAX_SORT.  Apply perm to every per-Gaussian array with
 * spin4d_permute_rows; decoding then returns attributes in sorted order.
 */
#define SPIN4D_MAX_SORT (1ll << 30)
size_t spin4d_morton_order_workspace(int64_t N);
int spin4d_morton_order(const spin4d_grid_desc* g, const float* pos, int64_t N, uint32_t* keys, uint32_t* perm,
                        void* workspace, size_t ws_bytes, spin4d_stream_t stream);

/*
 * dst row i = src row perm[i], i < N, rows of row_bytes bytes (a multiple of
 * 4).  src has src_rows rows; a row whose perm entry is not below src_rows
 * is left unwritten.  src and dst (device, 4-byte aligned, 16-byte aligned
 * for the vectorised path) must not overlap.
 */
int spin4d_permute_rows(const void* src, int64_t src_rows, void* dst, const uint32_t* perm, int64_t N,
                        int64_t row_bytes, spin4d_stream_t stream);

/*
 * Rendering of the decoded Gaussians (SPIN-4DGS section 3.1): each Gaussian
 * exp(-(x-mu)^T Sigma^-1 (x-mu)/2) (Eq. 1) is projected to the image with
 * Sigma_2D = J W Sigma W^T J^T (Eq. 3, W the view rotation, J the Jacobian
 * of the pinhole projection at the camera-space mean), and every pixel
 * blends the Gaussians covering it front to back,
 * C = sum_i c_i a_i prod_{j<i} (1 - a_j), a_i = o_i G_2D,i(pixel) (Eq. 4).
 *
 * Where the pages are silent the library fixes:
 *  - pixel (i, j) (column i, row j) is evaluated at image point
 *    (i + 1/2, j + 1/2); a camera-space point (x, y, z) maps to
 *    (fx x/z + cx, fy y/z + cy); Gaussians with z <= z_near are culled;
 *  - `lowpass` (pixels^2) is added to the diagonal of Sigma_2D (EWA's
 *    screen-space filter; 0 gives Eq. 3 exactly) and a Gaussian whose
 *    filtered Sigma_2D is not positive definite is culled;
 *  - a Gaussian covers a pixel when its Mahalanobis distance d^2 <= 9;
 *    a = min(alpha_max, o exp(-d^2/2)); a pixel skips a Gaussian with
 *    a < alpha_min; blending stops before the first Gaussian that would take
 *    the transmittance below t_stop; the remaining transmittance times
 *    `background` is added last;
 *  - order: camera depth z ascending (fp32), equal depths by index;
 *  - colour: sh_degree -1 reads RGB (N x 3); degree D in 0..3 reads
 *    (D+1)^2 real spherical-harmonic coefficients per channel,
 *    coefficient-major (N x 3(D+1)^2, value [n][3 (l*l + l + m) + channel]),
 *    evaluates the real SH without Condon-Shortley phase in the direction
 *    from the camera centre (-R^T t) to mu, and clamps the sum at 0.
 */
#define SPIN4D_MAX_IMAGE_SIDE 16384
#define SPIN4D_MAX_RENDER_GAUSSIANS (1ll << 31)
#define SPIN4D_MAX_RENDER_PAIRS (1ll << 31)

typedef struct spin4d_camera {
    float view[12];          /* world -> camera [R | t], row-major 3 x 4: x_c = R mu + t; looks along +z */
    float fx, fy, cx, cy;    /* pinhole intrinsics in pixels, fx, fy > 0 */
    int32_t width, height;   /* 1..SPIN4D_MAX_IMAGE_SIDE */
    float z_near;            /* > 0 */
} spin4d_camera;

typedef struct spin4d_render_desc {
    int32_t sh_degree;       /* -1 (RGB) or 0..3 */
    float lowpass;           /* >= 0, pixels^2 (e.g. 0.3) */
    float alpha_max;         /* in (0, 1) (e.g. 0.99) */
    float alpha_min;         /* in [0, alpha_max) (e.g. 1/255) */
    float t_stop;            /* in [0, 1) (e.g. 1e-4; 0 blends every covering Gaussian) */
    float background[3];
    int32_t mean_stride;     /* floats from one mean to the next: 3, or 4 for (x, y, z, t) rows */
    int32_t reserved;        /* must be 0 */
} spin4d_render_desc;

/*
 * Bytes of the render state for N Gaussians, an image of width x height and
 * room for max_pairs (Gaussian, 16x16 tile) pairs; 0 for invalid sizes.  The
 * state is owned by the caller (device, 256-byte aligned); the forward
 * fills it and the backward reads it.  Its first 8 bytes hold, after a
 * forward, the number of pairs the frame needed (uint64): a value above
 * max_pairs means the pairs did not fit, the image is incomplete and the call
 * must be repeated with a larger max_pairs.  Bytes 8..11 hold the pairs kept
 * (max_pairs when they did not fit; 0 if the total exceeds 2^32 - 1).
 */
size_t spin4d_render_state_bytes(int64_t N, int width, int height, int64_t max_pairs);

/*
 * Forward: means N rows of mean_stride floats (x, y, z first), cov N x 6
 * packed (xx, xy, xz, yy, yz, zz), opacity N, colours as sh_degree says (all
 * fp32, device, 4-byte aligned; may be NULL when N = 0).  Writes image
 * (3 x height x width fp32, channel planes) and, if final_T is not NULL, the
 * final transmittance (height x width fp32); both are overwritten, not
 * accumulated.  0 <= N <= SPIN4D_MAX_RENDER_GAUSSIANS.
 */
int spin4d_render_fwd(const spin4d_camera* cam, const spin4d_render_desc* desc, int64_t N, const float* means,
                      const float* cov, const float* opacity, const float* colours, float* image, float* final_T,
                      void* state, size_t state_bytes, int64_t max_pairs, spin4d_stream_t stream);

/*
 * Backward of spin4d_render_fwd for loss = sum(grad_image * image)
 * (grad_image 3 x height x width fp32): the same camera, desc, inputs,
 * state and max_pairs as the forward it follows.  ACCUMULATES into
 * grad_means (N x 3), grad_cov (N x 6, the gradient w.r.t. each packed
 * value), grad_opacity (N) and grad_colours (shaped like colours); any of
 * them may be NULL.  The culling, support, alpha_min and termination
 * decisions are those of the forward; a clamped alpha (o G > alpha_max) has
 * zero derivative.  Culled Gaussians get no gradient.
 */
int spin4d_render_bwd(const spin4d_camera* cam, const spin4d_render_desc* desc, int64_t N, const float* means,
                      const float* cov, const float* opacity, const float* colours, const float* grad_image,
                      void* state, size_t state_bytes, int64_t max_pairs, float* grad_means, float* grad_cov,
                      float* grad_opacity, float* grad_colours, spin4d_stream_t stream);

/*
 * Opt-in L2 residency for one buffer (the hash tables, say) on one stream:
 * the stream's access-policy window covers [base, base + bytes) with the
 * persisting property, and the current context's persisting-L2 set-aside
 * (cudaLimitPersistingL2CacheSize) is raised to the window's size, at most
 * cudaDevAttrMaxPersistingL2CacheSize.  Kernels later launched on `stream`
 * keep that range in L2 ahead of streaming data.  The library never sets a
 * window by itself.
 *   stream: a created stream (not NULL: the legacy stream takes no window).
 *   bytes is clipped to cudaDevAttrMaxAccessPolicyWindowSize; the clipped
 *   size goes to *applied_bytes when that is not NULL.
 * SPIN4D_ERR_UNSUPPORTED where the device has no persisting L2.
 * spin4d_l2_window_clear removes the stream's window, returns persisting
 * lines to normal (cudaCtxResetPersistingL2Cache) and restores the
 * context's set-aside to its value before the first spin4d_l2_window_set.
 * Both calls are host-synchronous configuration, not stream work.
 */
int spin4d_l2_window_set(spin4d_stream_t stream, const void* base, size_t bytes, size_t* applied_bytes);
int spin4d_l2_window_clear(spin4d_stream_t stream);

/*
 * 1 if this library was compiled with SPIN4D_CHECKED (libspin4d_checked.so),
 * else 0.  The checked build verifies on the device that every hash-table
 * index is below T and every HexPlane cell lies inside its plane; a failed
 * check is recorded and the access redirected to a valid address (nothing
 * traps), and spin4d_check_device_errors then returns SPIN4D_ERR_BOUNDS.
 */
int spin4d_checked_build(void);

/* Static string for a status code. */
const char* spin4d_status_string(int status);
/* cudaError_t of the last SPIN4D_ERR_CUDA returned on this thread (0 if none). */
int spin4d_last_cuda_error(void);
/* Library version, e.g. "0.1.0". */
const char* spin4d_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SPIN4D_H */
