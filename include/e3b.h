/*
 * e3b.h -- C ABI of the B200 (sm_100a) library for the channelwise ("uvu") Clebsch-Gordan
 * tensor product and the message-passing convolution built on it.
 *
 * Sources for what each call computes:
 *   [TP]   e3nn course, "Curriculum at a glance", lesson 03a (Clebsch-Gordan decomposition,
 *          parity rule p3 = p1 p2, triangle rule) and lesson 03b (weighted tensor product
 *          x (x)_w y, instructions, connection modes, counting weights).
 *   [IRR]  same page, lesson 02a (irreps strings "16x0e + 8x1o", memory layout); lesson 12a
 *          (mul_ir layout; a mismatch silently gives wrong numbers).
 *   [SH]   same page, lesson 02b (Y^l(R r) = D^l(R) Y^l(r), parity (-1)^l, normalisations);
 *          "Modular v2106 point models", Scope (component-normalised harmonics).
 *   [CONV] same course page, lesson 06a (point convolution m_ij = (R(|r_ij|) Y(r_ij)) (x)_w h_j,
 *          summed over neighbours) and lesson 05a (edge i -> j, r_ij = r_j - r_i);
 *          "Modular v2106 point models", Scope (1/sqrt(num_neighbors) normalisation);
 *          E3J (Peltre et al., "E3J: An Efficient and Open-Source Backend for Euclidean
 *          Equivariant Operations on GPU and TPU"), section E.2.2 (CSR receiver aggregation
 *          without atomics) and section C.2 (deterministic aggregation).
 *   [BWD]  E3J, section E.1 (reverse mode by transposing the linearised operation).
 *   [CG]   E3J, section G.2 (top-spin vector from a triangular system, then the lowering
 *          operator) -- the construction the library uses for its coefficient table.
 *
 * Conventions shared by every call
 *   - Tensors are dense, row-major, contiguous, in the mul_ir layout [IRR]: irrep blocks in
 *     order; inside a block [u][m] with m = -l..l fastest.  Every pointer must be 16-byte
 *     aligned.  The caller owns all memory; the library owns only plans.
 *   - Device pointers unless stated; every compute call is asynchronous on `stream` (a
 *     cudaStream_t passed as void*; NULL means the legacy default stream).
 *   - The element type of every float tensor is the plan's dtype (float or double).
 *   - Weights w are [B or E, weight_numel], path-major in instruction order, then channel u
 *     (uvu with mul_in2 = 1: one weight per (path, u)).  E3_W_SHARED: one row [weight_numel].
 *   - Real spherical harmonics use m = -l..l with the z axis as the pole and no
 *     Condon-Shortley phase, so Y^1 = sqrt(3) (y, z, x) / |r| under component normalisation.
 *   - Real CG tensors have Frobenius norm 1 per path; sign: positive C[0,0,0] when
 *     l1+l2+l3 is even, else a positive first nonzero entry in lexicographic (m1,m2,m3) order.
 *     1 (x) 1 then gives +dot/sqrt(3), +cross/sqrt(6) and the symmetric traceless product.
 *   - Path weight alpha_p defaults to sqrt((2 l3 + 1) / (mul_in2 * n_out)), n_out = number of
 *     instructions writing the same output block (uncollapsed: sqrt(2 l3 + 1)).
 *   - Errors are returned before any launch when they can be seen on the host; the message
 *     is available from e3_last_error().  Errors seen on the device (an index out of range,
 *     a bounded wait that gave up) are recorded in a status word: the plan's own for calls
 *     that take a plan (read and cleared by e3_plan_status()), one per device for the others
 *     (CSR, harmonics, radial network); e3_device_status() reads and clears the device's word
 *     and the words of every live plan on the device.  The offending edge is skipped, never
 *     dereferenced.
 *   - Results are deterministic: the same inputs give bitwise the same outputs (no atomics
 *     on floating-point data), except the uvw mode's grad_w and grad_y, which add partial sums
 *     with float atomics (their last bits may differ from run to run).
 *   - Per-device state (the status word, the coefficient tables, the address of the static CSR
 *     scratch) is set up on a device's first use and kept for the life of the process: after
 *     cudaDeviceReset, or after the primary context is destroyed, the library must not be called
 *     again in that process (the cached device addresses would be stale).
 */
#ifndef E3B_H
#define E3B_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define E3_API __attribute__((visibility("default")))
#else
#define E3_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  E3_OK = 0,
  E3_ERR_INVALID_ARG = 1,  /* NULL/misaligned pointer, negative size, bad enum */
  E3_ERR_IRREPS_PARSE = 2, /* malformed irreps string */
  E3_ERR_INSTRUCTION = 3,  /* triangle rule, parity rule, index range, multiplicity */
  E3_ERR_UNSUPPORTED = 4,  /* valid request with no compiled kernel (mode, degrees, layout) */
  E3_ERR_SHAPE = 5,        /* sizes that do not fit (e.g. row_ptr[N] != E, too many edges) */
  E3_ERR_INDEX = 6,        /* device: an index out of range was seen (checked kernels) */
  E3_ERR_CUDA = 7,         /* a CUDA runtime call failed */
  E3_ERR_TIMEOUT = 8       /* device: a bounded wait gave up */
} e3_status;

typedef enum { E3_F32 = 0, E3_F64 = 1 } e3_dtype;

/* Connection modes of lesson 03b [TP]: which channel indices an instruction ties.
 *   E3_UVU  out[u] = sum_v w[u,v] (x[u] (x) y[v])            tensor product and convolution
 *   E3_UUU  out[u] = w[u] (x[u] (x) y[u])                      tensor product only
 *   E3_UVW, E3_UUW                                             no kernels -> UNSUPPORTED */
typedef enum { E3_UVU = 0, E3_UVW = 1, E3_UUU = 2, E3_UUW = 3 } e3_mode;

/* SH normalisations of lesson 02b [SH]: component (sum_m Y^2 = 2l+1), integral
 * (component / sqrt(4 pi)), norm (component / sqrt(2l+1)).  Used only with edge vectors. */
typedef enum { E3_SH_COMPONENT = 0, E3_SH_INTEGRAL = 1, E3_SH_NORM = 2 } e3_sh_norm;

typedef enum { E3_W_PER_SAMPLE = 0, E3_W_SHARED = 1 } e3_weight_mode;

/* One instruction of lesson 03b [TP]: couple irrep i_in1 of input 1 with irrep i_in2 of
 * input 2 into irrep i_out of the output.  path_weight < 0 selects the default alpha_p. */
typedef struct {
  int32_t i_in1, i_in2, i_out;
  int32_t has_weight; /* must be 1 for the compiled kernels */
  double path_weight;
} e3_instruction;

typedef struct e3_plan e3_plan;

/* ---------------------------------------------------------------- plans (host, once) --- */

/* Build a plan [TP][IRR][CG].
 *   irreps_in1  node features, e.g. "64x0e+64x1o+64x2e".  Kernels need one irrep per degree
 *               l = 0..Lx in ascending order (any parities), one common multiplicity C with
 *               C % 4 == 0, Lx <= 3.
 *   irreps_in2  edge attributes, e.g. "1x0e+1x1o+1x2e+1x3o": multiplicity 1, l = 0..Ly, Ly <= 3.
 *               In the uuu mode the multiplicity is C (one y channel per x channel), and C
 *               may be any positive number.
 *   mode        E3_UVU or E3_UUU.  Weights per path: C (uvu with one y channel, one weight per
 *               (u, v)) or C (uuu, one per u); default alpha_p = sqrt((2 l3 + 1) / (fan * n_out))
 *               with fan = mul_in2 (uvu) or 1 (uuu), n_out = instructions writing the block.
 *   irreps_out  with n_instr == 0: a filter listing the output irreps allowed (multiplicities
 *               ignored; NULL or "" = all); instructions are then enumerated as
 *               for i1, for i2, for l3 = |l1-l2| .. l1+l2 with (l3, p1 p2) in the filter,
 *               each with its own output block of multiplicity C ("uncollapsed").
 *               With n_instr > 0: the output irreps that the instructions index.
 *   instr       n_instr explicit instructions (may be NULL when n_instr == 0).
 * The compiled kernels cover the full enumeration for (Lx, Ly, Lo) in the set listed by
 * e3_supported(); an explicit list must equal that enumeration (alphas may differ).
 * The CG table is generated here by the ladder construction and uploaded to the current
 * device on first use.  The plan is bound to the current CUDA device.
 * Returns IRREPS_PARSE, INSTRUCTION, UNSUPPORTED, INVALID_ARG or CUDA on failure. */
E3_API e3_status e3_plan_create(const char* irreps_in1, const char* irreps_in2, const char* irreps_out,
                         const e3_instruction* instr, int32_t n_instr, e3_mode mode,
                         e3_dtype dtype, e3_weight_mode wmode, e3_plan** plan);

E3_API e3_status e3_plan_destroy(e3_plan* plan);

/* Sizes per sample: dims of x, y, out (floats), weight_numel, number of paths.  Any output
 * pointer may be NULL. */
E3_API e3_status e3_plan_info(const e3_plan* plan, int64_t* dim_in1, int64_t* dim_in2, int64_t* dim_out,
                       int64_t* weight_numel, int32_t* n_paths);

/* The output irreps as a string ("64x0e+64x1o+...") written into buf (NUL-terminated);
 * *needed receives the length including the NUL.  buf may be NULL to query the length. */
E3_API e3_status e3_plan_irreps_out(const e3_plan* plan, char* buf, size_t buf_len, size_t* needed);

/* Per path: (l1, l2, l3) into lls[3*p..3*p+2] and alpha_p into alpha[p] (host arrays of
 * n_paths entries; either may be NULL). */
E3_API e3_status e3_plan_paths(const e3_plan* plan, int32_t* lls, double* alpha);

/* Synchronise `stream`, return the current device's status (E3_OK, E3_ERR_INDEX or
 * E3_ERR_TIMEOUT; the first error recorded since the last read by the calls without a plan or by
 * any live plan on the device) and clear it. */
E3_API e3_status e3_device_status(void* stream);

/* Synchronise `stream`, return the status word of `plan` (errors recorded by the kernels of calls
 * made with this plan since the last read) and clear it.  Calls on other plans, concurrent or not,
 * do not touch it; calls on this plan from several streams share it. */
E3_API e3_status e3_plan_status(const e3_plan* plan, void* stream);

/* Real CG table as generated for the plan's kernels: dense [2l1+1][2l2+1][2l3+1] doubles
 * for (l1, l2, l3), written to out (host).  Exposed for table-against-table checks. */
E3_API e3_status e3_cg_dense(int32_t l1, int32_t l2, int32_t l3, double* out);

/* Space-separated list "Lx,Ly,Lo ..." of degree triples with compiled kernels. */
E3_API const char* e3_supported(void);

/* ------------------------------------------------------------ tensor product (no graph) --- */

/* out[b] = TP(x[b], y[b], w[b]) for b < B [TP].
 *   x [B, dim_in1], y [B, dim_in2], w [B, weight_numel] (or [weight_numel] if shared),
 *   out [B, dim_out] (overwritten).  B == 0 is a no-op.  B < 2^31. */
E3_API e3_status e3_tp_forward(const e3_plan* plan, int64_t B, const void* x, const void* y,
                        const void* w, void* out, void* stream);

/* Bytes of device workspace that e3_tp_backward needs for n = B samples:
 * a ticket counter and one progress counter per work unit, which order the path groups of a
 * unit inside one launch.  The backward zeroes it on its stream before use. */
E3_API e3_status e3_backward_workspace_size(int64_t n, size_t* bytes);

/* Gradients of <grad_out, TP(x, y, w)> by transposition [BWD].  Each of grad_x [B, dim_in1],
 * grad_y [B, dim_in2], grad_w [B, weight_numel] may be NULL to skip it; outputs are
 * overwritten.  workspace: device buffer of at least e3_backward_workspace_size(B) bytes,
 * 16-byte aligned, owned by the caller and not used by any other call while this one runs
 * on its stream.  E3_W_SHARED plans are not supported for the backward. */
E3_API e3_status e3_tp_backward(const e3_plan* plan, int64_t B, const void* x, const void* y,
                         const void* w, const void* grad_out, void* grad_x, void* grad_y,
                         void* grad_w, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ harmonics --- */

/* Real spherical harmonics Y^0..Y^lmax of n vectors [SH]: out[i] = [Y^0 | Y^1 | ... ] with
 * (lmax+1)^2 values per vector, normalisation sh_norm; vec [n, 3] (any stride-3 layout,
 * element-aligned), out [n, (lmax+1)^2].  A zero vector gives Y^0 = 1 (scaled by the
 * normalisation) and Y^{l>0} = 0.  lmax <= 3.  n == 0 is a no-op. */
E3_API e3_status e3_spherical_harmonics(int32_t lmax, int64_t n, const void* vec, e3_sh_norm sh_norm,
                                 e3_dtype dtype, void* out, void* stream);

/* Gradient of the harmonics with respect to the vectors [SH]: for Y = the output of
 * e3_spherical_harmonics(lmax, n, vec, sh_norm),
 *   grad_vec[i] = sum_m grad_y[i, m] dY_m(vec_i)/dvec_i,
 * the chain rule that turns a gradient with respect to the harmonics (e3_conv_backward's grad_y)
 * into one with respect to edge vectors, hence positions: forces that conserve energy are the
 * negative gradient of the energy with respect to positions (e3nn course, "Curriculum at a
 * glance", lesson 07a).  Y depends on the direction only,
 * so grad_vec is orthogonal to vec and scales as 1/|vec|.  vec [n, 3], grad_y [n, (lmax+1)^2],
 * grad_vec [n, 3] (overwritten), element-aligned, of `dtype`; a zero vector gets a zero gradient.
 * lmax <= 3.  n == 0 is a no-op. */
E3_API e3_status e3_spherical_harmonics_backward(int32_t lmax, int64_t n, const void* vec, e3_sh_norm sh_norm,
                                          const void* grad_y, e3_dtype dtype, void* grad_vec, void* stream);

/* The backward of e3_spherical_harmonics_backward, so that forces can be trained through the
 * harmonics (xnn, "Run Models on Fused GPU Kernels", Training: the fast paths are twice
 * differentiable).  With grad_vec = J(vec)^T grad_y and u [n, 3] an upstream gradient for grad_vec:
 *   d_grad_y[i] = J(vec_i) u_i                          ([n, (lmax+1)^2]: derivative of Y along u)
 *   d_vec[i]    = grad over vec_i of grad_y_i . J(vec_i) u_i   ([n, 3]: a Hessian-vector product)
 * Both outputs overwritten; same layouts, dtype and limits as e3_spherical_harmonics_backward; a
 * zero vector gets zeros. */
E3_API e3_status e3_spherical_harmonics_double_backward(int32_t lmax, int64_t n, const void* vec, e3_sh_norm sh_norm,
                                                        const void* grad_y, const void* u, e3_dtype dtype,
                                                        void* d_grad_y, void* d_vec, void* stream);

/* ------------------------------------------------------------------ CSR segmentation --- */

/* Bytes of device workspace that e3_csr_build needs for N nodes and E edges. */
E3_API e3_status e3_csr_workspace_size(int64_t N, int64_t E, size_t* bytes);

/* Receiver and sender CSR of an edge list [CONV] (integer-only, bit-exact):
 *   perm_dst[E]      original edge ids in receiver order, ties in input order (stable);
 *   row_ptr_dst[N+1] node n's in-edges are positions row_ptr_dst[n] .. row_ptr_dst[n+1]-1;
 *   perm_src[E]      positions in receiver order, sorted stably by sender;
 *   row_ptr_src[N+1] node n's out-edges are perm_src[row_ptr_src[n] .. row_ptr_src[n+1]-1].
 * src, dst: int32 [E] in [0, N), or -1 for a padding edge (batches of fixed shape pad the edge
 * list; the E3J summary, sections 3.1.2 and 3.2, measures what padding edges that point to a
 * shared padding node cost).  An edge with -1 as sender or receiver belongs to no row: padding
 * edges follow the valid ones in both orders (input order among themselves), row_ptr_dst[N] and
 * row_ptr_src[N] count valid edges only, so no kernel walks them and E can stay fixed from step
 * to step.  Any other id out of range records E3_ERR_INDEX in the device status word
 * (e3_device_status) and the outputs are then unspecified.  workspace: device buffer of at least
 * e3_csr_workspace_size bytes, 256-byte aligned.  N, E < 2^31. */
E3_API e3_status e3_csr_build(int64_t N, int64_t E, const int32_t* src, const int32_t* dst,
                       int32_t* perm_dst, int32_t* row_ptr_dst, int32_t* perm_src,
                       int32_t* row_ptr_src, void* workspace, size_t ws_bytes, void* stream);

/* No counterpart in the paper: a library convenience.  Same result as e3_csr_build, but the
 * scratch lives in a fixed device array owned by the library, so the caller passes no
 * workspace and nothing is allocated.  It exists for callers that cannot allocate device
 * memory at the point where they build a graph: code running inside a CUDA stream capture
 * (cudaMalloc is not allowed there), code embedded in a host program whose device memory is
 * all owned by its own pool or arena, and loops that must avoid the implicit device
 * synchronisation of cudaMalloc / cudaFree.
 *   - Limit: E <= E3_CSR_STATIC_MAX_EDGES; larger E returns E3_ERR_SHAPE before any launch.
 *     The array (about 16.5 MiB) is held on every device that loads the library until exit.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     and sets up the device status word; make that first call before any stream capture.
 *   - Every call shares the one array: calls that overlap on the GPU (different streams, or
 *     different host threads without ordering) race and give undefined results.  Nothing in
 *     the array needs to start at zero: every pass overwrites what it reads.
 *   - Errors as e3_csr_build. */
#define E3_CSR_STATIC_MAX_EDGES (1 << 20)
E3_API e3_status e3_csr_build_static(int64_t N, int64_t E, const int32_t* src, const int32_t* dst,
                                     int32_t* perm_dst, int32_t* row_ptr_dst, int32_t* perm_src,
                                     int32_t* row_ptr_src, void* stream);

/* Rows of `in` gathered by `perm`: out[i, :] = in[perm[i], :] for i < n_rows, each row
 * row_bytes bytes (multiple of 4).  Used once per topology to put edge arrays into receiver
 * order.  perm entries must lie in [0, n_in_rows). */
E3_API e3_status e3_gather_rows(int64_t n_rows, int64_t n_in_rows, int64_t row_bytes,
                         const int32_t* perm, const void* in, void* out, void* stream);

/* Rows of `in` added into rows of `out`: out[idx[i], :] += in[i, :] for i < n_rows, each row
 * row_elems elements of `dtype`; out has n_out_rows rows.  The indices of one call must be
 * distinct (then no two threads touch one element and the result is deterministic).  This is the
 * reduction step of a sharded backward (E3J summary, section E.2.2: receiver-partitioned work):
 * a rank adds the grad_x partial rows other ranks computed for its senders, one source rank per
 * call, in a fixed order.  An index out of range records E3_ERR_INDEX and that row is skipped. */
E3_API e3_status e3_add_rows(int64_t n_rows, int64_t n_out_rows, int64_t row_elems, e3_dtype dtype,
                             const int32_t* idx, const void* in, void* out, void* stream);

/* ------------------------------------------------------------------- node reordering --- */

/* Sparse, irregular gathers bound message passing (Sobek: Streaming Equivariant Tensor Product
 * Convolutions, abstract); numbering nodes along a space-filling curve makes the senders of
 * neighbouring receivers neighbours in memory, so gathered rows are reused from L2.  The curve is
 * the Morton (Z-order) curve: each coordinate of pos[i] is quantised to 10 bits inside the box
 * [lo, lo + extent) (scale 1024 / extent in double, floor, clamped to [0, 1023]), bit b of axis k
 * goes to bit 3b + k of a 30-bit code, and perm[i] is the id of the node with the i-th smallest
 * code (stable: equal codes keep ascending ids; integer-only after the quantisation, bit-exact).
 * To renumber a graph: inv = inverse of perm; src, dst <- inv[src], inv[dst] (e3_remap_ids);
 * node rows <- rows[perm] (e3_gather_rows); results come back with rows[inv].
 *   pos [N, 3] of `dtype`; lo, extent: 3 host doubles (extent > 0); perm [N] int32 (device);
 *   workspace: device buffer of e3_morton_workspace_size(N) bytes, 256-byte aligned. */
E3_API e3_status e3_morton_workspace_size(int64_t N, size_t* bytes);
E3_API e3_status e3_morton_order(int64_t N, const void* pos, e3_dtype dtype, const double* lo,
                          const double* extent, int32_t* perm, void* workspace, size_t workspace_bytes,
                          void* stream);

/* inv[perm[i]] = i for a permutation perm of 0..N-1 (device int32 arrays).  Entries out of range
 * record E3_ERR_INDEX in the device status word and are skipped. */
E3_API e3_status e3_invert_permutation(int64_t N, const int32_t* perm, int32_t* inv, void* stream);

/* out[i] = map[ids[i]] for i < n, map of N entries (device int32 arrays; out may alias ids).  An id
 * out of [0, N) records E3_ERR_INDEX and gives -1. */
E3_API e3_status e3_remap_ids(int64_t n, const int32_t* ids, int64_t N, const int32_t* map, int32_t* out,
                       void* stream);

/* ------------------------------------------------------------------- radial network --- */

/* The per-edge path weights of the convolution as a learned function of the edge length (e3nn
 * course, "Curriculum at a glance", lesson 06a: m_ij = (R(|r_ij|) Y(r_ij)) (x)_w h_j; lesson 05b:
 * a Bessel basis times a polynomial envelope that keeps the energy smooth at the cutoff):
 *   f_n = sqrt(2/c) sin(n pi r / c) / r * u(r / c),  n = 1 .. n_basis  (r = |edge_vec|; r -> 0: limit)
 *   u(d) = 1 - (p+1)(p+2)/2 d^p + p (p+2) d^(p+1) - p (p+1)/2 d^(p+2) for d < 1, else 0
 *   w = SiLU(f W1) W2,  SiLU(x) = x / (1 + e^-x),  no biases.
 * The second layer ([E, hidden] x [hidden, n_out]) runs on the tensor cores (tcgen05, tf32 inputs
 * split into high and low parts, three passes, float32 accumulation: float32-level accuracy).
 * Float32 only.  W2 is first laid out once per weight update by e3_radial_prepare.
 *   hidden: a multiple of 8 in [8, 64]; n_out: a multiple of 4; n_basis in [1, 16]; p in [1, 32].
 *   edge_vec [E, 3], W1 [n_basis, hidden] row-major (device, 4-byte aligned); W2 [hidden, n_out]
 *   row-major (device); prep: device buffer of e3_radial_prep_size bytes, 16-byte aligned, owned
 *   by the caller; w [E, n_out] (device, 16-byte aligned, overwritten).  E == 0 is a no-op. */
E3_API e3_status e3_radial_prep_size(int32_t hidden, int32_t n_out, size_t* bytes);
E3_API e3_status e3_radial_prepare(int32_t hidden, int32_t n_out, const float* w2, void* prep, size_t prep_bytes,
                                   void* stream);
E3_API e3_status e3_radial_weights(int64_t E, const float* edge_vec, double cutoff, int32_t n_basis,
                                   int32_t envelope_p, int32_t hidden, const float* w1, const void* prep,
                                   int32_t n_out, float* w, void* stream);

/* ----------------------------------------------------------------------- convolution --- */

/* Work units of the convolution for one topology [CONV]: each receiver's in-edges (receiver CSR)
 * and each sender's out-edges (sender CSR) are cut into segments of at most 256 edges (one for a
 * row of <= 256 edges, also an empty one) -- the units the convolution's CTAs walk, so that a hub
 * does not serialise on one CTA.  Build once per topology, after e3_csr_build, and pass the
 * buffer to every e3_conv_forward / e3_conv_backward of that topology.  topo: device buffer of at
 * least e3_conv_topology_size(N, E) bytes, 16-byte aligned, owned by the caller.  A row pointer
 * out of range records E3_ERR_INDEX and gives that row no edges.  Integer-only. */
E3_API e3_status e3_conv_topology_size(int64_t N, int64_t E, size_t* bytes);
E3_API e3_status e3_conv_topology_build(int64_t N, int64_t E, const int32_t* row_ptr_dst,
                                 const int32_t* row_ptr_src, void* topo, size_t topo_bytes, void* stream);

/* The same units laid out in a processing order: order [N] (device int32) is a permutation of the
 * nodes, and the kernels then work through rows (receivers in the forward, senders in the
 * backward) in that order, each row's segments together and in segment order.  The numbering of
 * the nodes, and so every array's layout and every result, is unchanged (bitwise): only which
 * rows are in flight together changes.  With spatially random node ids and node rows larger than
 * L2, an order that follows space (e.g. e3_morton_order of the positions) makes the rows in flight
 * neighbours, so the x rows the forward gathers and the grad_out rows the backward gathers are
 * reused from L2 (Sobek: Streaming Equivariant Tensor Product Convolutions, abstract: sparse,
 * irregular gathers bound message passing).  An entry out of [0, N) records E3_ERR_INDEX and its
 * row gets no work; an order that is not a permutation gives unspecified results. */
E3_API e3_status e3_conv_topology_build_ordered(int64_t N, int64_t E, const int32_t* row_ptr_dst,
                                                const int32_t* row_ptr_src, const int32_t* order, void* topo,
                                                size_t topo_bytes, void* stream);

/* out[n] = out_scale * sum_{e : dst_e = n} TP(x[src_e], Y_e, w_e)   [CONV][TP]
 * Edge arrays are in receiver order (apply perm_dst once per topology):
 *   row_ptr_dst [N+1] (row_ptr_dst[0] == 0, non-decreasing; row_ptr_dst[N] <= E, the positions
 *   from row_ptr_dst[N] on being padding edges, which are not read);
 *   src [E] int32 in [0, N);
 *   exactly one of y [E, dim_in2] (given harmonics) or edge_vec [E, 3] (r_j - r_i, harmonics
 *   computed in registers with normalisation sh_norm; requires irreps_in2 = 1x0+1x1+..);
 *   w [E, weight_numel] (or [weight_numel] if shared); x [N, dim_in1]; out [N, dim_out]
 *   (overwritten; nodes without in-edges get zero rows).  E == 0 zero-fills out.
 * No floating-point atomics: each output row is reduced in edge order -- by one CTA, or, for a
 * row of more than 256 edges, by one CTA per 256-edge segment whose partial sums are added to the
 * row in segment order (a progress counter per row and path group orders them), so hubs do not
 * serialise and results stay bitwise repeatable.  topo: the buffer e3_conv_topology_build filled
 * for this row_ptr_dst (and the matching sender CSR).  workspace: device buffer of at least
 * e3_conv_workspace_size(plan, N, E) bytes, 16-byte aligned, owned by the caller and not used by
 * any other call while this one runs on its stream (the call zeroes it).  An src id out of range
 * records E3_ERR_INDEX in the device status word and that edge is skipped.  N, E < 2^31. */
E3_API e3_status e3_conv_workspace_size(const e3_plan* plan, int64_t N, int64_t E, size_t* bytes);
E3_API e3_status e3_conv_forward(const e3_plan* plan, int64_t N, int64_t E, const int32_t* row_ptr_dst,
                          const int32_t* src, const void* x, const void* y, const void* edge_vec,
                          e3_sh_norm sh_norm, const void* w, double out_scale, void* out,
                          const void* topo, void* workspace, size_t workspace_bytes, void* stream);

/* Gradients of <grad_out, conv_forward(...)> [BWD][CONV] with respect to
 *   grad_x [N, dim_in1]: sum over each node's out-edges (sender CSR: row_ptr_src, perm_src);
 *   grad_y [E, dim_in2]: per edge, with respect to the harmonics (also when they were
 *                        computed from edge_vec);
 *   grad_w [E, weight_numel]: per edge.
 * Any gradient pointer may be NULL to skip it.  Other arguments as e3_conv_forward; dst [E]
 * is the receiver of each (receiver-ordered) edge.  Padding positions (from row_ptr_dst[N] on)
 * get zero grad_y and grad_w rows.  Senders with more than 256 out-edges are split into
 * 256-edge segments like the forward's rows.  topo and workspace: as for e3_conv_forward.  No atomics on the gradients: the path groups of
 * a sender run in a fixed order, so results are bitwise repeatable.  A group that waits for
 * its predecessor longer than the wait limit (one second; e3_set_test_knobs) records
 * E3_ERR_TIMEOUT.  Shared weights are not
 * supported. */
E3_API e3_status e3_conv_backward(const e3_plan* plan, int64_t N, int64_t E, const int32_t* row_ptr_dst,
                           const int32_t* src, const int32_t* dst, const int32_t* row_ptr_src,
                           const int32_t* perm_src, const void* x, const void* y,
                           const void* edge_vec, e3_sh_norm sh_norm, const void* w,
                           const void* grad_out, double out_scale, void* grad_x, void* grad_y,
                           void* grad_w, const void* topo, void* workspace, size_t workspace_bytes,
                           void* stream);

/* No counterpart in the paper: failure-detection hooks for tests.  Every later convolution and
 * tensor-product launch in this process uses these values:
 *   wait_limit_ns  limit of every bounded device wait (a copy completion, a path group waiting
 *                  for its predecessor, a row segment waiting for the earlier ones); after it the
 *                  kernel records E3_ERR_TIMEOUT, stops waiting and returns normally.  0 restores
 *                  the default of one second.
 *   first_ticket   first ticket the ticketed kernels draw (default 0).  Raising it to k withholds
 *                  the first k work items of a launch (group-major order: group 0's units first),
 *                  so whatever waits for them times out: this is how a test makes a bounded wait
 *                  run out without faulting anything.  Results are then unspecified.
 * Process-global; not for concurrent use with production calls.  Negative values return
 * E3_ERR_INVALID_ARG. */
E3_API e3_status e3_set_test_knobs(int64_t wait_limit_ns, int32_t first_ticket);

/* Message of the last non-OK status returned on the calling thread ("" if none). */
E3_API const char* e3_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* E3B_H */
