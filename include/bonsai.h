/*
 * bonsai.h - C ABI of the B200 (sm_100a) weight-only low-bit linear layer.
 *
 * The operation.  A quantised weight is w[n,k] = s[n, k/128] * t[n,k], with
 * t in {-1,+1} (binary) or {-1,0,+1} (ternary) and one FP16 scale s per
 * group of 128 consecutive weights along the input dimension K
 * ("Cómo Bonsai Ternary 4B revoluciona la difusión texto-imagen", section
 * "Representación y almacenamiento de los pesos ternarios"; "Introducing
 * 1-bit and Ternary Bonsai Image 4B: Image Generation for Local Devices",
 * section "量化数学：1.125 和 1.71 是怎么来的").  The layer computes
 * out[m,n] = sum_k A[m,k] * w[n,k] for FP16 activations A and returns FP16.
 * Ternary codes are stored as INT2, two bits per weight ("Cómo Bonsai
 * Ternary 4B ...", same section); binary codes as one bit per weight (1.125
 * effective bits with the scale, "Introducing 1-bit and Ternary Bonsai
 * Image 4B ...", same section).
 *
 * Packed format (this library's own; the pages fix only the bit counts).
 * Rows of N, each a run of little-endian uint32 words along K.  Word j of a
 * row holds weights k = j*P .. j*P+P-1 (P = 32 binary, 16 ternary); local
 * weight i sits in pair p = i/2 of half h = i%2 (bits 0-15 or 16-31):
 *   binary : bit 16h + 15 - p; 1 means t = -1, 0 means t = +1;
 *   ternary: bits 16h + 14 - 2p (magnitude) and 16h + 15 - 2p (sign);
 *            t = 0 -> 00, t = +1 -> 01, t = -1 -> 11; 10 is not a code.
 * Base-3 ternary (BONSAI_TERNARY_B3, denser: 1.75 bits per weight against
 * INT2's 2): a row is a run of 112-byte blocks, one per 4 groups of 128
 * weights along K (28 * ceil(K/512) words); group 4b + r sits at byte
 * 112 b + 26 r; the block's last 8 bytes and group slots past the row's last
 * group are zero.  Byte j of a group holds the weights at group positions
 * j, j+26, j+52, j+78, j+104 as v = sum_i (t+1) 3^(4-i) (positions past 127
 * count as t+1 = 0), stored as the byte ceil(256 v / 243); the 13 other byte
 * values are not codes.
 * Scales: FP16 [N, K/128], row-major.  Activations: FP16 [M, K], row-major.
 * Output: FP16 [M, N], row-major.  FP16 values travel as uint16_t bits.
 *
 * Conventions for every call:
 *   - pointers are caller-owned DEVICE memory, 16-byte aligned, on the
 *     current CUDA device, unless a parameter says host;
 *   - `stream` is a cudaStream_t (NULL = legacy default stream); work is
 *     enqueued on it and the call returns before it finishes, unless noted;
 *   - the library allocates no device memory;
 *   - the return value is a bonsai_status; on any error nothing is launched
 *     (argument errors) or the CUDA error is reported as BONSAI_ERR_CUDA;
 *   - shapes: M >= 0, N >= 0, K >= 0 with K a multiple of 128 (no partial
 *     groups); zero-sized problems are valid no-ops.
 */
#ifndef BONSAI_H_
#define BONSAI_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BONSAI_BINARY = 1,       /* t in {-1,+1}, 1 bit per weight */
  BONSAI_TERNARY_INT2 = 2, /* t in {-1,0,+1}, 2 bits per weight */
  BONSAI_TERNARY_B3 = 3    /* t in {-1,0,+1}, five per byte: 1.75 bits per weight */
} bonsai_mode;

typedef enum {
  BONSAI_OK = 0,
  BONSAI_ERR_INVALID_ARG = 1, /* unknown mode, null pointer with a non-empty shape */
  BONSAI_ERR_SHAPE = 2,       /* negative size, K not a multiple of 128, size overflow */
  BONSAI_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  BONSAI_ERR_BAD_CODE = 4,    /* bonsai_pack met a code outside the alphabet */
  BONSAI_ERR_CUDA = 5,        /* a CUDA runtime call failed */
  BONSAI_ERR_ARCH = 6,        /* the current device is not sm_100 */
  BONSAI_ERR_TIMEOUT = 7      /* a kernel gave up a bounded wait (see bonsai_get_device_error) */
} bonsai_status;

/* Bytes of packed weights for an [N,K] weight: N*K/8 (binary), N*K/4
 * (INT2 ternary) or N*112*ceil(K/512) (base-3 ternary).  Returns 0 for an
 * invalid mode or shape. */
size_t bonsai_packed_bytes(int64_t N, int64_t K, int mode);

/* Bytes of the FP16 scales for an [N,K] weight: 2*N*K/128. */
size_t bonsai_scale_bytes(int64_t N, int64_t K);

/* Pack weight codes.  The alphabets and bit counts come from the pages:
 * ternary t in {-1,0,+1} stored as INT2, two bits per weight, for CUDA ("Cómo
 * Bonsai Ternary 4B revoluciona la difusión texto-imagen", section
 * "Representación y almacenamiento de los pesos ternarios"); binary t in
 * {-1,+1} at one bit, 1.125 effective bits per weight with the group scale
 * ("Bonsai Image 4B 1-bit untuk pembuatan gambar di perangkat lokal",
 * section "Bonsai Image 4B untuk pembuatan gambar lokal").  The bit layout
 * is this library's.
 * codes: int8 [N,K] with every value in the mode's alphabet; packed:
 * bonsai_packed_bytes(N,K,mode) bytes, written in the format above.  This
 * call is offline (once per weight): it synchronises `stream` before
 * returning so that it can report BONSAI_ERR_BAD_CODE when a code is outside
 * the alphabet (packed is then unspecified).  Concurrent
 * bonsai_pack calls on different streams share the flag that reports it. */
int bonsai_pack(const int8_t* codes, int64_t N, int64_t K, int mode, void* packed, void* stream);

/* Exact dequantisation: w[n,k] = fp16(t[n,k] * s[n,k/128]), the IEEE
 * product (bit-exact: +-s, +-0, or NaN for 0*inf and NaN scales).  This is
 * the pages' weight equation w_i = scale_g * t_i with one FP16 scale per
 * group of 128 weights ("Cómo Bonsai Ternary 4B revoluciona la difusión
 * texto-imagen", section "Representación y almacenamiento de los pesos
 * ternarios").
 * packed: as written by bonsai_pack; scales: FP16 [N,K/128]; w: FP16 [N,K].
 * Meant for testing and for callers that want a dense copy. */
int bonsai_dequant(const void* packed, const uint16_t* scales, int64_t N, int64_t K, int mode,
                   uint16_t* w, void* stream);

/* The fused low-bit GEMM: out[m,n] = fp16( sum_k A[m,k] * w[n,k] ).
 * This is the quantised linear layer of the pages: every matmul-heavy linear
 * of the diffusion transformer (Q/K/V projections, MLP weights, the
 * double-stream add-K/Q/V linears) holds such weights ("Cómo Bonsai Ternary
 * 4B revoluciona la difusión texto-imagen", section "Representación y
 * almacenamiento de los pesos ternarios"), and the transformer runs once per
 * denoising step, so its weight bandwidth sets the step's speed
 * ("Introducing 1-bit and Ternary Bonsai Image 4B: Image Generation for
 * Local Devices", section "端侧约束：为什么 diffusion transformer 是唯一值得压缩的部分").
 * A: FP16 [M,K]; packed/scales: as above for an [N,K] weight; out: FP16
 * [M,N].  Products are formed exactly and summed in FP32 on the tensor
 * cores, then rounded once to FP16 (nearest even).  Scales must be finite
 * with |s| < 32768 for INT2 ternary weights (the kernel forms 2*s*t in
 * FP16); outside that range the result is unspecified.  out must not
 * overlap A, packed or scales.  An INT2 field with the pattern 10 (not a
 * ternary code) contributes zero; a base-3 byte that is not a code gives
 * unspecified values for its five weights.
 * Stream order: A is read, and out written, only after everything enqueued
 * before the call on `stream` has completed.  packed and scales, however, are
 * read-only weights and may be read as soon as the launch starts, which for
 * M <= 16 overlaps the end of the kernel enqueued just before it: that
 * kernel must not write packed or scales (work enqueued earlier may; so may
 * bonsai_pack, which returns only after its writes are complete). */
int bonsai_lowbit_gemm(const uint16_t* A, const void* packed, const uint16_t* scales, int64_t M,
                       int64_t N, int64_t K, int mode, uint16_t* out, void* stream);

/* The same GEMM with the activations and the output in host memory (the
 * pages' layer applied to a batch that lives on the host; no counterpart of
 * its own on the pages).  A_host: FP16 [M,K]; out_host: FP16 [M,N]; both
 * should be page-locked (cudaHostAlloc / pinned) for the copies to overlap.
 * packed/scales: device memory as for bonsai_lowbit_gemm.  A_dev and
 * out_dev: caller-owned device work buffers of at least M*K and M*N FP16
 * values, 16-byte aligned (the library allocates nothing).
 * The rows are split into chunks of a multiple of 256; chunk c's
 * host->device copy, GEMM and device->host copy run on three library-owned
 * streams, so that the copies in both directions overlap the GEMMs of other
 * chunks.  The work is ordered after everything already enqueued on `stream`
 * and everything enqueued on `stream` afterwards is ordered after it; the
 * call returns without synchronising.  Host buffers must stay valid and
 * unmodified (A_host) / unread (out_host) until `stream` reaches that point.
 * Concurrency: every call on one device uses the same three library streams
 * (and one process-wide lock while it enqueues), so calls made from several
 * threads or user streams run one after another on the GPU, never
 * overlapped with each other.
 * Errors: as bonsai_lowbit_gemm, plus BONSAI_ERR_INVALID_ARG for null
 * pointers. */
int bonsai_lowbit_gemm_host(const uint16_t* A_host, const void* packed, const uint16_t* scales, int64_t M,
                            int64_t N, int64_t K, int mode, uint16_t* out_host, uint16_t* A_dev,
                            uint16_t* out_dev, void* stream);

/* One problem of bonsai_lowbit_gemm_batch: out = A * w^T for an [N,K]
 * weight, with the operands, layouts and rules of bonsai_lowbit_gemm. */
typedef struct {
  const uint16_t* A;      /* FP16 [M,K], device */
  const void* packed;     /* packed [N,K] weight (bonsai_pack), device */
  const uint16_t* scales; /* FP16 [N,K/128], device */
  uint16_t* out;          /* FP16 [M,N], device */
  int64_t M, N, K;
} bonsai_gemm_problem;

/* Several independent low-bit GEMMs in one call, all of one weight mode
 * (no counterpart of its own on the pages; it serves their bandwidth-bound
 * case: at a few tokens a quantised linear is a stream of its packed
 * weights, and the weight bytes of the transformer's linears per denoising
 * step set its speed, "Introducing 1-bit and Ternary Bonsai Image 4B: Image
 * Generation for Local Devices", section "端侧约束：为什么 diffusion
 * transformer 是唯一值得压缩的部分").
 * Problems with M <= 16 run together in persistent launches of up to 96
 * problems each: one CTA per SM walks the 128-row weight tiles of all of
 * them, so the weight stream does not stop between problems for a launch,
 * a dependency release and a tail of its own.  Problems with M > 16 are
 * launched one by one, as bonsai_lowbit_gemm launches them.  Each result
 * is the one bonsai_lowbit_gemm gives up to the order of the FP32 sums (the
 * same accuracy).
 * problems: HOST array of `count` entries, read during the call only.
 * Independence: no problem's out may overlap any A, packed, scales or out
 * of the batch; the order of the launches is unspecified.
 * Stream order: as for bonsai_lowbit_gemm (the weights of the first problems
 * may be read while the kernel enqueued just before still runs).
 * Errors: every problem is checked before anything is launched and the
 * first error found is returned; BONSAI_ERR_INVALID_ARG also for count < 0
 * or a NULL problems with count > 0. */
int bonsai_lowbit_gemm_batch(const bonsai_gemm_problem* problems, int count, int mode, void* stream);

/* ------------------------------------------ 4-bit group-affine weights --
 * The pages name "4-bit HQQ" for the text encoder ("Cómo Bonsai Ternary 4B
 * revoluciona la difusión texto-imagen", section "Arquitectura de despliegue
 * y eficiencia en tiempo de ejecución") and nothing more.  This library
 * reads it as HQQ's published scheme: an unsigned 4-bit q per weight and, per
 * group of 64 weights along K, an FP16 scale s and an FP16 zero z, the weight
 * being w = fp16(fp16(q - z) * s) (two IEEE FP16 operations).  The group
 * size and the packing are this library's choices.
 * Packed: rows of K/8 little-endian uint32 words; word j holds k = 8j..8j+7,
 * weight i of it at bit 16 (i%2) + 4 (i/2) (weights 2p, 2p+1 at the same
 * offset of the two 16-bit halves).  scales, zeros: FP16 [N, K/64].
 * K must be a multiple of 128. */

/* Bytes of packed 4-bit weights: N*K/2 (0 for an invalid shape). */
size_t bonsai_hqq4_packed_bytes(int64_t N, int64_t K);

/* q: uint8 [N,K] with values 0..15 -> packed.  Offline; synchronises
 * `stream` to report BONSAI_ERR_BAD_CODE for a value above 15. */
int bonsai_hqq4_pack(const uint8_t* q, int64_t N, int64_t K, void* packed, void* stream);

/* Exact dequantisation: w = fp16(fp16(q - z) * s), FP16 [N,K] (bit-exact,
 * IEEE rules for NaN, infinities and signed zeros). */
int bonsai_hqq4_dequant(const void* packed, const uint16_t* scales, const uint16_t* zeros, int64_t N, int64_t K,
                        uint16_t* w, void* stream);

/* out[m,n] = fp16( sum_k A[m,k] * w[n,k] ) with the weights above, formed
 * exactly as bonsai_hqq4_dequant forms them and summed in FP32 on the tensor
 * cores; the same tiling, split and error behaviour as bonsai_lowbit_gemm.
 * Weights that come out infinite or NaN give unspecified outputs. */
int bonsai_hqq4_gemm(const uint16_t* A, const void* packed, const uint16_t* scales, const uint16_t* zeros, int64_t M,
                     int64_t N, int64_t K, uint16_t* out, void* stream);

/* The launch bonsai_lowbit_gemm makes for this problem on the current
 * device: *block_t = tokens per tile (the MMA's N; each tile also covers 128
 * weight rows), *ksplit = CTAs that share one tile along K as a thread-block
 * cluster (1 = no split), *ctas = CTAs launched, *tiles = output tiles.
 * ctas < tiles x ksplit means the persistent form: one CTA per SM walks the
 * tiles tau = blockIdx, blockIdx + ctas, ...  Host-side only (queries
 * occupancy, launches nothing).  Zero-sized problems report zeros.  mode 4
 * asks for the launch of bonsai_hqq4_gemm. */
int bonsai_gemm_plan(int64_t M, int64_t N, int64_t K, int mode, int* block_t, int* ksplit, int* ctas,
                     int* tiles);

/* Reads and clears the device-side error word of the current device: 0 if
 * no kernel reported a problem since the last call, else a bonsai_status
 * (BONSAI_ERR_TIMEOUT when a bounded wait inside a kernel ran out; the
 * kernel then returned early and its output is unspecified).  Synchronises
 * the device. */
int bonsai_get_device_error(void);

/* Human-readable name of a status code (static string). */
const char* bonsai_status_string(int status);

/* Self-test of the bounded-wait path: launches one kernel that waits on an
 * mbarrier nobody arrives at, with a limit of `limit_ns` nanoseconds, and
 * returns what the kernel recorded: BONSAI_ERR_TIMEOUT when the wait gave up
 * as designed.  Clears the device error word before and after. */
int bonsai_selftest_wait_timeout(uint64_t limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* BONSAI_H_ */
