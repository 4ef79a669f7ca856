/*
 * qml.h -- C ABI of libqml: batched state-vector simulation of a
 * hardware-efficient ansatz (HEA) with a fused forward pass that ends in <Z0>
 * and a fused adjoint backward pass that yields every parameter gradient, on
 * NVIDIA B200 (sm_100a).
 *
 * The method follows the five web summaries of Kawase, "Fast and
 * memory-efficient classical simulation of quantum machine learning via
 * forward and backward gate fusion" (arXiv 2603.02804).  Citations below name
 * the page and its section:
 *   [Deep-dive]  blog "深度解析：正向与反向门融合驱动的高效量子机器学习仿真"
 *                (hugo-pages-80e.pages.dev), sections 1.2, 1.3, 1.4, 2.1, 2.3, 3.2
 *   [Gist-EN]    gist.science "Fast and memory-efficient classical simulation
 *                of quantum machine learning via forward and backward gate
 *                fusion", Technical Summary sections 2 and 4
 *   [Gist-ES]    gist.science/es, Resumen tecnico section 2
 *
 * Circuit (qubit q = bit q of the amplitude index, R_P(t) = exp(-i t P/2)):
 *   |0...0>  ->  Ry(x[b][q]) on every qubit (angle encoding)
 *   for l in 0..L-1:  Rx(theta[l][q][0]) Ry(theta[l][q][1]) Rz(theta[l][q][2])
 *                     on every qubit q, then CZ(q, q+1) for q = 0..n-2
 *   E[b] = <psi_b| Z0 |psi_b>
 *
 * Conventions for every call:
 *   - Complex arrays are interleaved (re, im) float32 pairs, 8-byte aligned;
 *     state vectors are [B][2^n] complex, i.e. B * 2^n * 2 floats.
 *   - Every pointer named *_dev is device memory owned by the caller; the
 *     library never allocates device memory itself (no cudaMalloc, no
 *     allocating library routine).  *_host pointers are host memory (pinned
 *     memory makes the copies asynchronous).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *   - Calls are asynchronous on `stream` unless stated otherwise.  Argument
 *     errors are returned synchronously and nothing is launched.  Device-side
 *     problems (a non-finite expectation value, a failed bounds check) are
 *     latched in a status word inside the workspace and returned by the next
 *     qml_sync().
 *   - No call aborts, traps or throws across the ABI.
 *   - A context is not thread-safe; concurrent calls on one context race.
 */
#ifndef QML_H
#define QML_H

#include <stddef.h>

#if defined(__GNUC__)
#define QML_API __attribute__((visibility("default")))
#else
#define QML_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QML_OK = 0,
  QML_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, size out of range */
  QML_ERR_UNSUPPORTED = 2,  /* configuration outside what the kernels handle */
  QML_ERR_WORKSPACE = 3,    /* no workspace set, or too small for this batch */
  QML_ERR_CUDA = 4,         /* a CUDA runtime call failed */
  QML_ERR_CKPT_MISMATCH = 5,/* checkpoint slot / batch / storage mismatch */
  QML_ERR_NUMERIC = 6,      /* a non-finite value was produced */
  QML_ERR_BOUNDS = 7,       /* a device-side bounds check failed */
  QML_ERR_TIMEOUT = 8       /* reserved: a bounded device wait gave up */
} qml_status;

/* Storage format of checkpoint slots: fp32 (re, im) pairs, or the
 * memory-save mode's bfloat16 pairs (round to nearest even; compute stays
 * fp32 or fp64).  [Gist-EN] Technical Summary sec. 2 "Memory-Saving Mode";
 * [Deep-dive] sec. 2.3.  fp64 pairs only for contexts of qml_create_f64. */
typedef enum { QML_STORE_FP32 = 0, QML_STORE_BF16 = 1, QML_STORE_FP64 = 2 } qml_storage;

typedef struct {
  int n_qubits;       /* 1 .. 30 */
  int n_layers;       /* 1 .. 100000 */
  int max_batch;      /* largest B any call will use, >= 1 */
  int ckpt_block;     /* layers per checkpoint block (0 = no checkpoints);
                         the pages find 10-20 best, [Deep-dive] sec. 2.3 */
  qml_storage storage;
} qml_config;

typedef struct qml_ctx qml_ctx; /* opaque, host-side metadata only */

/* Version of the ABI (currently 1). */
QML_API int qml_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
QML_API const char* qml_status_str(qml_status s);

/* Create a context for one circuit shape on CUDA device `device`.  Builds the
 * host-side pass schedule; touches no device memory.  *out is NULL on error.
 * Fault injection for tests of the error paths, read from the environment at
 * creation (all on the host; no device fault is ever provoked):
 *   QML_FAULT=alloc         qml_set_workspace returns QML_ERR_WORKSPACE
 *   QML_FAULT=ckpt_corrupt  every forward pass leaves its checkpoint slots
 *                           unrecorded: the backward pass returns
 *                           QML_ERR_CKPT_MISMATCH
 *   QML_FAULT=nan_theta     the first rotation's coefficients are NaN in
 *                           every forward pass (fp64 contexts: the first
 *                           angle, in a copy of theta inside the workspace),
 *                           with any entangler: qml_sync returns
 *                           QML_ERR_NUMERIC */
QML_API qml_status qml_create(const qml_config* cfg, int device, qml_ctx** out);

/* Destroy a context.  The caller frees the workspace afterwards. */
QML_API qml_status qml_destroy(qml_ctx* ctx);

/* Device workspace bytes that calls with batch B need: the pass schedule,
 * gate-coefficient tables, checkpoint slots for max_batch samples, reduction
 * partials and the status word.  Returns 0 for B out of range. */
QML_API size_t qml_workspace_bytes(const qml_ctx* ctx, int B);

/* Hand the context a caller-owned device workspace (256-byte aligned,
 * qml_workspace_bytes(ctx, max_batch) bytes).  The schedule is uploaded on
 * `stream`; the status word is cleared. */
QML_API qml_status qml_set_workspace(qml_ctx* ctx, void* ws_dev, size_t bytes, void* stream);

/* Angle encoding only: psi_dev[b] = (x) Ry(x[b][q])|0>, the product state the
 * forward pass starts from ([Deep-dive] sec. 1.2: psi in C^{2^n}).
 *   x_dev    [B][n] float32
 *   psi_dev  [B][2^n] complex64, written */
QML_API qml_status qml_init_state_encode(qml_ctx* ctx, const float* x_dev, int B, float* psi_dev,
                                 void* stream);

/* Fused forward pass.  Builds the encoded state, applies every layer in
 * passes that each read and write the state once ([Deep-dive] sec. 1.4 item
 * 1; [Gist-EN] sec. 2 "Forward Path Gate Fusion"), writes checkpoint slots at
 * block boundaries, and reduces E = <psi|Z0|psi> ([Deep-dive] sec. 1.2,
 * E(theta); sec. 3.2, matrix-free expectation).
 *   theta_dev  [L][n][3] float32 (Rx, Ry, Rz angle per qubit per layer)
 *   x_dev      [B][n] float32 encoding angles
 *   psi_dev    [B][2^n] complex64, out: final state (16-byte aligned: for
 *              n > 12 the passes load their tiles with tensor copies)
 *   expect_dev [B] float32, out */
QML_API qml_status qml_forward_expect(qml_ctx* ctx, const float* theta_dev, const float* x_dev, int B,
                              float* psi_dev, float* expect_dev, void* stream);

/* Fused adjoint backward pass.  Starting from the final state and
 * lambda = dL/dE[b] * Z0 psi, walks the passes in reverse; inside each pass
 * it rebuilds psi_{j-1} = U_j^dagger psi_j on chip alongside
 * lambda_{j-1} = U_j^dagger lambda_j and accumulates
 * dL/dtheta_j = 2 Re<lambda_j| dU_j/dtheta_j |psi_{j-1}>
 * ([Deep-dive] sec. 1.2 adjoint-gradient equation and lambda recursion,
 * sec. 1.4 item 2; [Gist-EN] sec. 2 "Backward Path Gate Fusion").  At each
 * checkpoint boundary psi is reloaded from its slot.  Gradients are reduced in
 * a fixed order (deterministic).
 *   psi_dev     [B][2^n] complex64: in, the final state from
 *               qml_forward_expect; clobbered (used as working memory)
 *   lambda_dev  [B][2^n] complex64 working memory, clobbered
 *   (psi_dev and lambda_dev 16-byte aligned, as for the forward pass)
 *   dLdE_dev    [B] float32, dL/dE per sample
 *   grad_dev    [L][n][3] float32, out (overwritten): sum_b dL/dE[b] dE[b]/dtheta
 * theta_dev must hold the angles of the forward call that produced psi_dev
 * (the gradient is that circuit's); when it is the same buffer as in the
 * context's last forward call, with no setter in between, the gate tables
 * that call prepared for both directions are reused. */
QML_API qml_status qml_backward_adjoint(qml_ctx* ctx, const float* theta_dev, const float* x_dev, int B,
                                float* psi_dev, float* lambda_dev, const float* dLdE_dev,
                                float* grad_dev, void* stream);

/* Loss seed for L = mean_b (E[b] - y[b])^2: g[b] = 2 (E[b] - y[b]) / B and
 * loss = L (one float).  Any of g_dev / loss_dev may be NULL. */
QML_API qml_status qml_loss_seed(qml_ctx* ctx, const float* expect_dev, const float* y_dev, int B,
                         float* g_dev, float* loss_dev, void* stream);

/* Store psi (standard layout) into checkpoint slot `slot` (0 ..
 * qml_num_ckpt_slots-1) in the context's storage format, or restore it.  A
 * restore from a slot last written with a different batch size or by nothing
 * returns QML_ERR_CKPT_MISMATCH.  ([Gist-EN] sec. 2 "Gradient Checkpointing
 * Integration": only block-boundary states are stored.) */
QML_API qml_status qml_ckpt_save(qml_ctx* ctx, int slot, const float* psi_dev, int B, void* stream);
QML_API qml_status qml_ckpt_restore(qml_ctx* ctx, int slot, float* psi_dev, int B, void* stream);

/* Number of checkpoint slots the schedule uses (ceil(L / ckpt_block) - 1). */
QML_API int qml_num_ckpt_slots(const qml_ctx* ctx);

/* Standalone Z0 expectation of B states: E[b] = sum_i |psi_b(i)|^2 (+1 if
 * bit 0 of i is 0, else -1).  [Deep-dive] sec. 3.2 (matrix-free Pauli
 * expectation, Z part). */
QML_API qml_status qml_expect_z0(qml_ctx* ctx, const float* psi_dev, int B, float* expect_dev,
                         void* stream);

/* Largest number of CZ bonds in an entangler. */
#define QML_MAX_BONDS 1024

/* Entangler for the following forward and backward calls: every layer ends
 * with CZ(bonds[2e], bonds[2e+1]) for e = 0 .. n_bonds-1 (host array of
 * n_bonds pairs of distinct qubits).  The default after qml_create is the
 * chain CZ(q, q+1), q = 0 .. n-2 ([Deep-dive] sec. 2.1 names CZ entanglers
 * without a topology; the open chain is the plain reading).  CZ gates are diagonal, so any bond
 * graph (ring, all-to-all, brick, none: n_bonds = 0) runs through the same
 * fused passes; a bond listed twice cancels (CZ^2 = I).  Returns
 * QML_ERR_INVALID_ARG on a bad pair or count (the previous entangler then
 * stays in force).  Set it before the forward pass whose backward it serves. */
QML_API qml_status qml_set_entangler(qml_ctx* ctx, int n_bonds, const int* bonds);

/* Number of bonds (CZ) or pairs (CNOT) of the entangler in force. */
QML_API int qml_entangler_bonds(const qml_ctx* ctx);

/* CNOT entanglers for the following forward and backward calls: every layer
 * ends with CNOT(pairs[2e] -> pairs[2e+1]) (control, target) for e = 0 ..
 * n_pairs-1 in list order, e.g. the ladder (q, q+1).  The pages name CNOT
 * gates as the other entangler their kernels fuse by recomputing indices
 * ([Deep-dive] sec. 3.2).  A layer's CNOT list is a linear map M of the
 * index bits over GF(2).  Contexts of 13..20 qubits (two qubit sets A, B)
 * whose map factors as M = M2 M1, M1 changing only A's bits and M2 only B's
 * (true whenever the A-to-A block of M is invertible, e.g. the ladder or the
 * ring), run fused: M1 and M2 are applied inside the rotation passes, as a
 * permutation of each tile's positions (fp32: while the tile is read or in a
 * layout exchange; fp64: in the shared-memory tile), and each layer costs two
 * passes with no gather through HBM.  Other contexts (other sizes,
 * re-uploading, maps that do not factor)
 * run each layer's rotations as the fused passes of a one-layer schedule and
 * then one gather pass into a second state buffer (the workspace grows by B
 * * 2^n complex64, or complex128 in fp64).  Either way the schedule changes:
 * if a workspace was set before, it is released by this call and must be set
 * again (qml_workspace_bytes / qml_set_workspace); the compute calls return
 * QML_ERR_WORKSPACE until then.  Checkpoint slots, observables and
 * re-uploading apply as with CZ, in both precisions.  QML_ERR_INVALID_ARG on
 * a bad pair or count.  qml_set_entangler switches back to CZ (and releases
 * the workspace the same way when the fused schedule was in force). */
QML_API qml_status qml_set_entangler_cnot(qml_ctx* ctx, int n_pairs, const int* pairs);

/* Kind of the entangler in force: 0 CZ, 1 CNOT (-1 for NULL). */
QML_API int qml_entangler_kind(const qml_ctx* ctx);

/* Debugging aid (host only): the CNOT layer map as images of single index
 * bits, written like qml_debug_schedule (returns the number of ints, -1 when
 * the entangler is not CNOT).  Layout: [n, then n images of M (the layer
 * sends the amplitude at b to M b) on qubit bits, n images of M^-1, then the
 * same two maps on working-state address bits, then 1 if the fused schedule
 * is in force (else 0), then n images of M1 and n images of M2 on qubit bits
 * (M = M2 M1; zeros when not fused)]. */
QML_API int qml_debug_entangler_map(const qml_ctx* ctx, int* out, int cap);

/* Data re-uploading for the following forward and backward calls: with
 * on != 0 every layer starts with the angle encoding Ry(x[b][q]) on every
 * qubit again (no parameters; its inverse is un-applied in the backward pass,
 * which then needs x_dev).  Off after qml_create.  QML_ERR_UNSUPPORTED for
 * n_qubits < 5.  Set it before the forward pass whose backward it serves. */
QML_API qml_status qml_set_reupload(qml_ctx* ctx, int on);
QML_API int qml_reupload(const qml_ctx* ctx);

/* 1 when the context's passes run in split form, 0 when they apply fused
 * SU(2) rotations, -1 for a null context.  The split form (fp32 contexts
 * without re-uploading or CNOT entanglers) rewrites every fused rotation
 * U = Rz(g) Ry(b) Rx(a) exactly as Rz(phi1) Ry(vt) Rz(phi2), applies the real
 * Ry in tangent form and merges each layer's Rz factors with its CZ bonds
 * into one diagonal (Deep-dive blog sec. 1.4, forward and backward gate
 * fusion: the gates are fused differently, the results are the same up to
 * rounding).  Informational: every entry point gives the same results either
 * way. */
QML_API int qml_split_form(const qml_ctx* ctx);

/* Measurement aid (not part of the simulation): the FMA throughput of the
 * current device, for the ALU rooflines of the pass kernels.  One launch of
 * independent FMA chains over every SM, `iters` steps of 8 chains per thread,
 * timed with CUDA events on `stream` (the call synchronises).  fp64 != 0:
 * DFMA; otherwise the packed f32x2 FMA of the fp32 kernels.  *tflops =
 * 2 x FMAs / time (TFLOP/s); *ms (optional) = the launch's duration.
 * Allocates nothing. */
QML_API qml_status qml_measure_fma_peak(int fp64, int iters, void* stream, double* tflops, float* ms);

/* Largest number of Pauli-string terms an observable may have. */
#define QML_MAX_OBS_TERMS 4096

/* Observable for the following forward, backward and expectation calls:
 * O = sum_k coeffs[k] P_k, a sum of Pauli strings (the general observable O
 * of E(theta) = <psi|O|psi> and lambda_M = dL/dE O psi_M, [Deep-dive] sec.
 * 1.2; evaluated matrix-free by bit flips, [Deep-dive] sec. 3.2, the
 * expectation listing).
 *   n_terms  0 .. QML_MAX_OBS_TERMS; 0 restores the default O = Z0
 *   paulis   host, n_terms * n_qubits characters (no terminator): character
 *            k * n_qubits + q is the factor of term k on qubit q, one of
 *            'I', 'X', 'Y', 'Z'
 *   coeffs   host, n_terms finite real coefficients
 * The context keeps a copy; the terms reach the device workspace at the next
 * call that needs them (a copy from pageable memory on that call's stream,
 * which may wait for the stream: make that call before capturing a graph).
 * Returns QML_ERR_INVALID_ARG on a bad letter, a non-finite coefficient or a
 * bad count; the previous observable then stays in force. */
QML_API qml_status qml_set_observable(qml_ctx* ctx, int n_terms, const char* paulis, const double* coeffs);

/* Number of terms of the observable in force (0 = the default Z0). */
QML_API int qml_observable_terms(const qml_ctx* ctx);

/* Standalone expectation of the observable in force: E[b] = <psi_b|O|psi_b>
 * for B states in the standard layout (fp64 partial sums, deterministic). */
QML_API qml_status qml_expect_observable(qml_ctx* ctx, const float* psi_dev, int B, float* expect_dev,
                                         void* stream);

/* Allocation-free Z0 expectation, for callers that may not allocate device
 * memory at all (for example a plugin inside an application whose framework
 * owns all device memory through its own pool, or a loop in which an
 * allocation that may synchronise the device is not allowed).  It needs no
 * context and no workspace: the partial sums of its two-stage reduction live
 * in a fixed array compiled into the library (32768 doubles = 256 KiB, held
 * on every GPU that loads the library until the process exits).  It computes
 * exactly what qml_expect_z0 computes; the paper has no counterpart of this
 * entry point.
 *   psi_dev    [B][2^n] complex64 on the current device (8-byte aligned)
 *   expect_dev [B] float32, out
 * Limits and behaviour:
 *   - B * ceil(2^n / 65536) must not exceed 32768 (e.g. B <= 2048 at n = 20,
 *     B <= 4 at n = 29); larger calls return QML_ERR_WORKSPACE and launch
 *     nothing.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it; make
 *     that first call before any stream capture.  The cache is tied to the
 *     device's CUDA context: the first call after a cudaDeviceReset looks the
 *     address up again (so it, too, belongs before any capture).
 *   - All calls on a device share the one array.  Each call overwrites every
 *     partial it later reads, so stale contents are never used, but calls
 *     whose kernels overlap on the GPU (different streams, no ordering) race
 *     on it.
 *   - No status word: a non-finite expectation is written to expect_dev as
 *     it is, and nothing is latched for a later qml_sync.
 *   - No cudaMalloc, cudaFree or allocating library routine is called. */
QML_API qml_status qml_expect_z0_static(const float* psi_dev, int n_qubits, int B, float* expect_dev,
                                        void* stream);

/* One full training step through HOST buffers: copies x, theta and y from
 * host to device, runs qml_forward_expect, qml_loss_seed and
 * qml_backward_adjoint, and copies E, the loss and the gradient back.  Needs
 * the larger workspace of qml_host_workspace_bytes (it also holds psi, lambda
 * and the staged inputs).  Synchronises `stream` before returning.
 *   x_host [B][n], theta_host [L][n][3], y_host [B]      (in)
 *   expect_host [B], loss_host [1], grad_host [L][n][3]  (out; may be NULL
 *   except grad_host)
 * Repeated calls: once a call with the same host buffers, batch and
 * workspace has run, the next such call captures the step's copies and
 * launches into a CUDA graph (on a stream of the context's own) and later
 * ones replay it on `stream`, which removes the per-launch host cost of small
 * circuits.  The buffers' contents are read at each replay, so new inputs in
 * the same buffers are fine.  Any setter (entangler, observable,
 * re-uploading, workspace) and timing (qml_enable_timing) return it to the
 * eager path; a step that cannot be captured (e.g. pageable host buffers on
 * some systems) stays eager.  Host buffers should be pinned. */
QML_API size_t qml_host_workspace_bytes(const qml_ctx* ctx, int B);
QML_API qml_status qml_step_host(qml_ctx* ctx, const float* x_host, const float* theta_host,
                         const float* y_host, int B, float* expect_host, float* loss_host,
                         float* grad_host, void* stream);

/* Synchronise `stream` and return the first device-side error latched since
 * the last qml_sync / qml_set_workspace (then clear it). */
QML_API qml_status qml_sync(qml_ctx* ctx, void* stream);

/* Pass-kernel timing, for benchmarks.  While enabled, every
 * qml_forward_expect / qml_backward_adjoint call records one CUDA event pair
 * on its own stream around its pass-kernel launches (events are host-side
 * handles; no device memory is allocated).  qml_read_timing waits for those
 * events and returns the summed milliseconds and launch counts since the
 * previous read (any output pointer may be NULL). */
QML_API qml_status qml_enable_timing(qml_ctx* ctx, int enable);
QML_API qml_status qml_read_timing(qml_ctx* ctx, double* fwd_pass_ms, long long* fwd_pass_launches,
                                   double* bwd_pass_ms, long long* bwd_pass_launches);

/* Number of kernels this context has launched so far (host-side counter). */
QML_API long long qml_launch_count(const qml_ctx* ctx);

/* Schedule introspection (host only, no device work): the pass plan as a flat
 * int array, for tests of the scheduler.  Writes at most `cap` ints into
 * `out` and returns the number needed.  Layout: [n_passes, then per pass:
 * rotated-set id, encodes (0/1), last (0/1), checkpoint slot (-1 = none),
 * n_ops, then per op 4 ints (kind, a, b, c)].  Op kinds:
 * 1 = register-layout exchange (a = from layout, b = to layout),
 * 2 = rotate (a = layer, b = bit mask of the rotated qubits, c = first slot),
 * 3 = CZ ladder (a = layer), 4 = encode (a = layout). */
QML_API int qml_debug_schedule(const qml_ctx* ctx, int* out, int cap);

/* Debugging aid: the memory view of pass `pass` (0-based, forward order),
 * written like qml_debug_schedule (returns the number of ints, -1 on a bad
 * argument).  Layout: [tensor-copy loads (0/1), then 5 dimensions x
 * (kind, lowest qubit, qubits, first bit in the out-of-tile index), then 12
 * tile bits x (qubit or -1 - unit bit, element offset in the copied tile),
 * then n_out, then the out-of-tile qubits (in address order), then the
 * working-state address bit of each tile bit (-1 for a unit bit) and of each
 * out-of-tile qubit, then the register-layout variant].  Dimension kinds: 0
 * unused, 1 in-tile address bits (copied whole), 2 out-of-tile address bits
 * (fixed per tile), 3 sample, 4 out-of-tile address bits merged with the
 * sample index above them.  The lowest address bit of a run is given. */
QML_API int qml_debug_tile_view(const qml_ctx* ctx, int pass, int* out, int cap);

/* Debugging aid: the kernels' register layouts, written like
 * qml_debug_schedule.  Layout: for phase 0..2 and layout variant 0..1, the
 * tile bit of each of the 7 thread-index bits then of each of the 5
 * register-index bits; then the 12 shared-memory slot weights of the tile
 * bits (slot of a position = sum of the weights of its set bits) and the
 * number of slots of the 16-byte exchanges; then the same two for the 8-byte
 * exchanges of the passes that load tiles by tensor copies. */
QML_API int qml_debug_layouts(int* out, int cap);

/* ------------------------------------------------------------------------
 * fp64 compute mode.  The pages state that the simulator runs in double as
 * well as single precision ([Gist-EN] Technical Summary sec. 2 and 4).  A
 * context made by qml_create_f64 runs the same schedule of fused forward and
 * adjoint backward passes with complex128 state vectors and fp64 arithmetic;
 * its inputs and outputs are float64 and its state vectors are [B][2^n]
 * (re, im) double pairs, 16-byte aligned.  Checkpoint slots take the
 * config's storage: QML_STORE_FP64 keeps them exact, QML_STORE_FP32 /
 * QML_STORE_BF16 round them (the backward pass then restarts from the
 * rounded state at each slot).  CZ and CNOT entanglers, data re-uploading
 * (qml_set_reupload, any n) and Pauli-sum observables (qml_set_observable,
 * evaluated in fp64) apply.
 * The fp32 calls (qml_forward_expect, qml_backward_adjoint, qml_loss_seed,
 * qml_step_host, qml_init_state_encode, qml_ckpt_save / _restore,
 * qml_expect_z0, qml_expect_observable) return QML_ERR_UNSUPPORTED on an
 * fp64 context, and the calls below on an fp32 one.  Workspace, entangler,
 * timing and sync calls are shared.
 * ------------------------------------------------------------------------ */

/* Create an fp64 context (same arguments and errors as qml_create). */
QML_API qml_status qml_create_f64(const qml_config* cfg, int device, qml_ctx** out);

/* 32 or 64: the arithmetic precision of a context (-1 for NULL). */
QML_API int qml_precision(const qml_ctx* ctx);

/* As qml_forward_expect, in fp64.
 *   theta_dev [L][n][3] float64, x_dev [B][n] float64
 *   psi_dev   [B][2^n] complex128, out: final state (16-byte aligned)
 *   expect_dev [B] float64, out */
QML_API qml_status qml_forward_expect_f64(qml_ctx* ctx, const double* theta_dev, const double* x_dev, int B,
                                          double* psi_dev, double* expect_dev, void* stream);

/* As qml_backward_adjoint, in fp64 (psi_dev and lambda_dev complex128,
 * 16-byte aligned, both clobbered; dLdE_dev [B] and grad_dev [L][n][3]
 * float64).  Gradients are reduced in a fixed order (deterministic). */
QML_API qml_status qml_backward_adjoint_f64(qml_ctx* ctx, const double* theta_dev, const double* x_dev, int B,
                                            double* psi_dev, double* lambda_dev, const double* dLdE_dev,
                                            double* grad_dev, void* stream);

/* As qml_loss_seed, in fp64. */
QML_API qml_status qml_loss_seed_f64(qml_ctx* ctx, const double* expect_dev, const double* y_dev, int B,
                                     double* g_dev, double* loss_dev, void* stream);

/* As qml_step_host, in fp64 (host arrays of doubles; the workspace of
 * qml_host_workspace_bytes, which for an fp64 context sizes the staged
 * buffers in doubles). */
QML_API qml_status qml_step_host_f64(qml_ctx* ctx, const double* x_host, const double* theta_host,
                                     const double* y_host, int B, double* expect_host, double* loss_host,
                                     double* grad_host, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QML_H */
