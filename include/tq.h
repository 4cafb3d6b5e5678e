/*
 * tq.h -- C ABI of the 3DTurboQuant vector codec in libw4a4 (sm_100a).
 *
 * Source: page "3DTurboQuant: Training-Free Near-Optimal Quantization for 3D
 * Reconstruction Models" (gist.science), technical summary:
 *   [TQ-FLOW] section 2.2: separate the norm gamma = ||theta||, rotate the unit
 *             direction with a random orthogonal matrix Pi, quantize every
 *             coordinate to a b-bit index with a codebook precomputed for the
 *             coordinates' Beta distribution; reconstruct gamma * Pi^T * c[index].
 *   [TQ-BETA] section 2.1: after the rotation a coordinate of a d-dimensional unit
 *             vector follows the density (d - 3)/2-power law
 *             f(x) ~ (1 - x^2)^((d-3)/2) on [-1, 1]; Lloyd-Max quantizers of it.
 *   [TQ-KV]   section 4.2: the DUSt3R KV cache, d = 1024, b = 4.
 * Readings: the page's Pi is the Q factor of a Gaussian matrix (tq_rotation_qr,
 * tq_encode_dense, tq_decode_dense below); tq_encode / tq_decode are a fast
 * variant with Pi = H diag(s) / sqrt(d), H the natural-order Hadamard matrix and
 * s a caller-given +-1 vector (an orthogonal matrix applied in O(d log d), not
 * the page's); code = number of boundaries strictly below the coordinate; two
 * 4-bit codes per byte, element 2i in the low nibble.
 *
 * Supported: d = 1024, b = 4 (W4A4_ERR_UNSUPPORTED otherwise).  Status codes,
 * stream and alignment conventions are those of w4a4.h: device pointers owned by
 * the caller, 16-byte aligned, calls enqueue on `stream` and return.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stdint.h>

#include "w4a4.h"

#ifdef __cplusplus
extern "C" {
#endif

/* [TQ-BETA] Lloyd-Max codebook of the coordinate density for dimension d and b
 * bits, computed on the host in double precision and rounded to fp32:
 * centroids [2^b] and boundaries [2^b - 1] (HOST arrays), both increasing and
 * odd-symmetric (the middle boundary is 0). */
w4a4_status tq_codebook(int32_t d, int32_t b, float *centroids, float *boundaries);

/* [TQ-FLOW] encode n vectors X [n, d] (fp32, row-major): norms [n] = ||x||
 * (fp32), codes [n, d/2] = the 4-bit indices of y = Pi x / ||x|| against
 * boundaries [15] (device copy of tq_codebook's).  signs [d]: the +-1 entries of
 * s (device, fp32).  A zero vector gets norm 0 and the codes of y = 0.  Decisions
 * in binary32: (H diag(s) x)_j is compared with boundary_k * ||x|| * sqrt(d). */
w4a4_status tq_encode(const float *X, int64_t n, int32_t d, const float *signs,
                      const float *boundaries, uint8_t *codes, float *norms, void *stream);

/* [TQ-FLOW] decode: Y [n, d] (fp32) = norms[i] * Pi^T * centroids[codes[i, :]],
 * centroids [16] on the device. */
w4a4_status tq_decode(const uint8_t *codes, const float *norms, int64_t n, int32_t d,
                      const float *signs, const float *centroids, float *Y, void *stream);

/* ---------------------------------------------------------------------------
 * The page's rotation: Pi is the random orthogonal matrix from the QR
 * factorisation of a Gaussian matrix ([TQ-FLOW]), applied as a dense matrix
 * product on the tensor cores.  (tq_encode / tq_decode above are the fast
 * variant with the signed Hadamard matrix in its place.)
 * ------------------------------------------------------------------------- */

/* [TQ-FLOW] Pi = Q diag(sign(diag R)) for the Householder QR factorisation
 * G = Q R of the d x d matrix G (HOST, row-major, double; independent standard
 * normal entries for the page's random rotation): the sign fix makes the
 * factorisation unique (R with a positive diagonal).  Outputs, HOST arrays of
 * d * d floats, row-major: pi_hi / pi_lo, Pi split into two tf32 terms (hi =
 * the binary32 value with its 13 low mantissa bits cleared, lo = the rest
 * rounded to tf32; hi + lo is within 2^-22 of Pi), and pit_hi / pit_lo, the
 * same for Pi^T.  Copy them to the device for tq_encode_dense (pi_*) and
 * tq_decode_dense (pit_*).  d = 1024 only (W4A4_ERR_UNSUPPORTED otherwise).
 * Computed in double precision on the calling thread: about a second. */
w4a4_status tq_rotation_qr(const double *G, int32_t d, float *pi_hi, float *pi_lo, float *pit_hi,
                           float *pit_lo);

/* [TQ-FLOW] encode with the dense Pi: norms [n] = ||x|| (fp32), codes
 * [n, d/2] = the 4-bit indices of y = Pi x / ||x|| against boundaries [15]
 * (device copy of tq_codebook's; the decision t_k < y is taken as
 * t_k ||x|| < (Pi x)_k in binary32, the product in tf32 with three terms).
 * pi_hi, pi_lo: device copies of tq_rotation_qr's.  A zero vector gets norm 0
 * and codes 7 (y = 0). */
w4a4_status tq_encode_dense(const float *X, int64_t n, int32_t d, const float *pi_hi, const float *pi_lo,
                            const float *boundaries, uint8_t *codes, float *norms, void *stream);

/* [TQ-FLOW] decode with the dense Pi: Y [n, d] (fp32) = norms[i] Pi^T
 * centroids[codes[i, :]]; pit_hi, pit_lo: device copies of tq_rotation_qr's
 * Pi^T terms; centroids [16] on the device. */
w4a4_status tq_decode_dense(const uint8_t *codes, const float *norms, int64_t n, int32_t d,
                            const float *pit_hi, const float *pit_lo, const float *centroids, float *Y,
                            void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
