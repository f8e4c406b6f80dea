/*
 * kvq_oracle.c -- plain, slow, obviously-correct CPU oracle for the rotated
 * INT2 KV-cache hot path (rotate -> quantize -> append, and decode attention
 * over the packed cache).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file.  Only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * generator with the CUDA library: every formula below is written out again
 * from the method description and from the cache-format specification.
 *
 * What the method computes (sources are the pages on the subject):
 *   - "Output-Aware Rotation for INT2 KV-Cache Quantization", section
 *     "Key Details": each head has an orthogonal rotation, applied to the
 *     cache before INT2 quantization and removed after the attention
 *     computation.  Section "Why It Matters": the inference (attention)
 *     kernel itself is unchanged.
 *   - "RotateKV: Accurate and Robust 2-Bit KV Cache Quantization ..."
 *     abstract, item (i): the rotation is a channel reordering followed by a
 *     fast Walsh-Hadamard transform; item (ii): that rotation applied to the
 *     keys before RoPE and across a group of heads; item (iii): attention
 *     sinks, singled out by massive activations, are protected from 2-bit
 *     quantization.
 *   - "KVLinC : KV Cache Quantization with Hadamard Rotation and Linear
 *     Correction", abstract: a Hadamard rotation of the values, and
 *     lightweight linear correction adapters that compensate for the errors
 *     the quantized keys introduce (decode_one's adapter, below).
 * The pages fix the 2-bit width only.  The group of 32 along head_dim, the
 * asymmetric min/max grid with an fp16 scale and fp16 zero per group, and the
 * packed cache layout are this library's format; they are restated here as
 * the format specification describes them.
 *
 * Precision: rotations and attention in fp64; the quantizer in exact IEEE
 * fp32 with no contraction (build with -ffp-contract=off, no fast-math).
 *
 * Parity pins for every function are in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define D 128      /* head_dim */
#define GS 32      /* quantization group size along head_dim */
#define NG 4       /* groups per row */
#define BLK_TOK 16 /* tokens per cache block */
#define BLK_BYTES 1536

/* status bits (same meaning as the library's device status word) */
#define ST_CAPACITY 1
#define ST_BAD_LEN 2

/* ------------------------------------------------------------------------ */
/* IEEE binary16 <-> binary32, written from the IEEE 754 encoding.            */
/* ------------------------------------------------------------------------ */

/* binary32 -> binary16, round to nearest, ties to even; overflow -> +-inf. */
uint16_t orc_f32_to_f16(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t ax = x & 0x7fffffffu;
    if (ax >= 0x7f800000u) {                   /* inf / nan */
        if (ax == 0x7f800000u) return (uint16_t)(sign | 0x7c00u);
        return (uint16_t)(sign | 0x7e00u);     /* quiet nan */
    }
    if (ax >= 0x477ff000u) return (uint16_t)(sign | 0x7c00u); /* >= 65520 */
    if (ax >= 0x38800000u) {                   /* half normal range */
        uint32_t e = (ax >> 23) - 127u + 15u;
        uint32_t m = ax & 0x7fffffu;
        uint32_t hm = m >> 13, rem = m & 0x1fffu;
        uint32_t h = (e << 10) | hm;
        if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u;
        return (uint16_t)(sign | h);
    }
    if (ax <= 0x33000000u) return (uint16_t)sign; /* <= 2^-25 -> 0 */
    {                                          /* half subnormal */
        uint32_t e = ax >> 23;                 /* 102..112 */
        uint32_t m = (ax & 0x7fffffu) | 0x800000u;
        uint32_t shift = 126u - e;             /* 14..24 */
        uint32_t hm = m >> shift;
        uint32_t rem = m & ((1u << shift) - 1u);
        uint32_t half = 1u << (shift - 1u);
        if (rem > half || (rem == half && (hm & 1u))) hm += 1u;
        return (uint16_t)(sign | hm);
    }
}

float orc_f16_to_f32(uint16_t h) {
    uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
    uint32_t e = ((uint32_t)h >> 10) & 0x1fu;
    uint32_t m = (uint32_t)h & 0x3ffu;
    uint32_t x;
    if (e == 0x1fu) {
        x = sign | 0x7f800000u | (m << 13);
    } else if (e != 0) {
        x = sign | ((e - 15u + 127u) << 23) | (m << 13);
    } else if (m == 0) {
        x = sign;
    } else {                                   /* subnormal: m * 2^-24 */
        float v = (float)m * 5.9604644775390625e-08f;
        memcpy(&x, &v, 4);
        x |= sign;
    }
    float f;
    memcpy(&f, &x, 4);
    return f;
}

/* ------------------------------------------------------------------------ */
/* Rotations (fp64).                                                          */
/* ------------------------------------------------------------------------ */

/* In-place unnormalised Walsh-Hadamard transform in Sylvester (natural)
 * order: H[i][j] = (-1)^popcount(i & j).  Butterfly (a, b) -> (a+b, a-b)
 * at strides 1, 2, 4, ... n/2.  RotateKV abstract, item (i) (FWHT). */
void orc_fwht_f64(double *y, int n) {
    for (int s = 1; s < n; s <<= 1)
        for (int i = 0; i < n; i++)
            if ((i & s) == 0) {
                double a = y[i], b = y[i + s];
                y[i] = a + b;
                y[i + s] = a - b;
            }
}

/* x_rot = x . R (row-vector convention, R row-major R[i][j]), or in FWHT
 * mode x_rot = FWHT(y)/sqrt(128) with y[i] = x[perm[i]] (channel reordering
 * then Hadamard; RotateKV item (i), KVLinC abstract).  fp64 throughout. */
static void rotate_f64(const double *x, int mode, const float *R,
                       const int32_t *perm, double *out) {
    if (mode == 0) {
        for (int j = 0; j < D; j++) {
            double acc = 0.0;
            for (int i = 0; i < D; i++) acc += x[i] * (double)R[i * D + j];
            out[j] = acc;
        }
    } else {
        for (int i = 0; i < D; i++) out[i] = x[perm[i]];
        orc_fwht_f64(out, D);
        double sc = 1.0 / sqrt((double)D);
        for (int i = 0; i < D; i++) out[i] *= sc;
    }
}

/* Inverse rotation, o . R^T (the rotation "removed after the attention
 * computation", OptR page, "Key Details").  FWHT mode: y = FWHT(o)/sqrt(128),
 * out[perm[i]] = y[i]. */
static void unrotate_f64(const double *o, int mode, const float *R,
                         const int32_t *perm, double *out) {
    if (mode == 0) {
        for (int i = 0; i < D; i++) {
            double acc = 0.0;
            for (int j = 0; j < D; j++) acc += o[j] * (double)R[i * D + j];
            out[i] = acc;
        }
    } else {
        double y[D];
        for (int i = 0; i < D; i++) y[i] = o[i];
        orc_fwht_f64(y, D);
        double sc = 1.0 / sqrt((double)D);
        for (int i = 0; i < D; i++) out[perm[i]] = y[i] * sc;
    }
}

/* fp64 rotation of fp64 rows, exported for the invariance pins. */
void orc_rotate_f64_rows(const double *x, int64_t n, int mode, const float *R,
                         const int32_t *perm, double *out) {
    for (int64_t r = 0; r < n; r++) rotate_f64(x + r * D, mode, R, perm, out + r * D);
}

void orc_unrotate_f64_rows(const double *o, int64_t n, int mode, const float *R,
                           const int32_t *perm, double *out) {
    for (int64_t r = 0; r < n; r++) unrotate_f64(o + r * D, mode, R, perm, out + r * D);
}

/* Rotate fp16 rows into "the rotated fp32 input" of the quantizer: fp64
 * rotation of the exactly widened fp16 row, rounded once to fp32. */
void orc_rotate_rows_f32(const uint16_t *x, int64_t n, int mode, const float *R,
                         const int32_t *perm, float *out) {
    double xin[D], xo[D];
    for (int64_t r = 0; r < n; r++) {
        for (int i = 0; i < D; i++) xin[i] = (double)orc_f16_to_f32(x[r * D + i]);
        rotate_f64(xin, mode, R, perm, xo);
        for (int i = 0; i < D; i++) out[r * D + i] = (float)xo[i];
    }
}

/* ------------------------------------------------------------------------ */
/* INT2 quantizer (exact fp32).                                              */
/* ------------------------------------------------------------------------ */

/* One row of 128 rotated fp32 values -> 128 codes in {0,1,2,3} and, per group
 * of 32 consecutive elements, an fp16 scale s and fp16 zero z:
 *   mn, mx = min, max of the group
 *   s = half(fp32((mx - mn) / 3)),  z = half(mn)       (a zero is stored +0)
 *   inv = (s == 0) ? 0 : fp32(1 / float(s))
 *   c = clamp(rint_even(fp32(fp32(x - float(z)) * inv)), 0, 3)
 * Dequantised value: c * s + z.  Four levels = INT2 (OptR page, intro and
 * "Key Details"; RotateKV abstract, "2-bit"). */
void orc_quantize_row(const float *x, uint8_t *codes, uint16_t *s_out, uint16_t *z_out) {
    for (int g = 0; g < NG; g++) {
        const float *xg = x + g * GS;
        float mn = xg[0], mx = xg[0];
        for (int e = 1; e < GS; e++) {
            if (xg[e] < mn) mn = xg[e];
            if (xg[e] > mx) mx = xg[e];
        }
        float r = mx - mn;
        float sf = r / 3.0f;
        uint16_t s = orc_f32_to_f16(sf + 0.0f);
        uint16_t z = orc_f32_to_f16(mn + 0.0f);
        float sF = orc_f16_to_f32(s), zF = orc_f16_to_f32(z);
        float inv = (sF == 0.0f) ? 0.0f : 1.0f / sF;
        for (int e = 0; e < GS; e++) {
            float d = xg[e] - zF;
            float t = d * inv;
            float rt = rintf(t);
            int c = (rt < 0.0f) ? 0 : (rt > 3.0f ? 3 : (int)rt);
            codes[g * GS + e] = (uint8_t)c;
        }
        s_out[g] = s;
        z_out[g] = z;
    }
}

void orc_quantize_rows(const float *x, int64_t n, uint8_t *codes, uint16_t *s, uint16_t *z) {
    for (int64_t r = 0; r < n; r++)
        orc_quantize_row(x + r * D, codes + r * D, s + r * NG, z + r * NG);
}

/* Logical packing, 4 codes per byte: the code of element j goes to byte
 * (j mod 32), bits 2*(j div 32) .. 2*(j div 32)+1.  So byte e carries the
 * element e of each of the 4 groups. */
void orc_pack_row(const uint8_t *codes, uint8_t *bytes) {
    for (int e = 0; e < 32; e++) {
        uint8_t b = 0;
        for (int g = 0; g < NG; g++) b |= (uint8_t)((codes[g * GS + e] & 3u) << (2 * g));
        bytes[e] = b;
    }
}

void orc_unpack_row(const uint8_t *bytes, uint8_t *codes) {
    for (int j = 0; j < D; j++) codes[j] = (uint8_t)((bytes[j % 32] >> (2 * (j / 32))) & 3u);
}

/* ------------------------------------------------------------------------ */
/* Physical cache block (16 tokens, 1536 bytes), restated from the format     */
/* specification.  tau = token index in the block, r = tau mod 8,             */
/* th = tau div 8.                                                            */
/*   K codes  [0,512):    logical 32-bit word wi (bytes 4wi..4wi+3) at        */
/*                        16*(4r + wi%4) + 4*(2*th + wi/4)                    */
/*   V codes  [512,1024): token pair p = tau/2, side = tau%2; logical 16-bit  */
/*                        piece w (bytes 2w, 2w+1) at                         */
/*                        512 + 16*(4*(w%8) + p%4) + 4*(2*(p/4) + w/8) + 2*side*/
/*   K meta   [1024,1280): group g {s, z} (two fp16, s first) at              */
/*                        1024 + 8*(4r + g) + 4*th                            */
/*   V meta   [1280,1536): group g {s, z} (two fp16, s first) at              */
/*                        1280 + 8*(4r + g) + 4*th                            */
/* ------------------------------------------------------------------------ */

static size_t off_kword(int tau, int wi) {
    int r = tau % 8, th = tau / 8;
    return (size_t)(16 * (4 * r + wi % 4) + 4 * (2 * th + wi / 4));
}
static size_t off_vpiece(int tau, int w) {
    int p = tau / 2, side = tau % 2;
    return (size_t)(512 + 16 * (4 * (w % 8) + p % 4) + 4 * (2 * (p / 4) + w / 8) + 2 * side);
}
static size_t off_kmeta(int tau, int g) {
    int r = tau % 8, th = tau / 8;
    return (size_t)(1024 + 8 * (4 * r + g) + 4 * th);
}
static size_t off_vmeta(int tau, int g) {
    int r = tau % 8, th = tau / 8;
    return (size_t)(1280 + 8 * (4 * r + g) + 4 * th);
}

static void put16(uint8_t *p, uint16_t v) { p[0] = (uint8_t)(v & 0xff); p[1] = (uint8_t)(v >> 8); }
static uint16_t get16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* Store one token's packed K and V rows and their metadata into a block. */
void orc_store_token(uint8_t *block, int tau, const uint8_t *kbytes, const uint8_t *vbytes,
                     const uint16_t *ks, const uint16_t *kz, const uint16_t *vs,
                     const uint16_t *vz) {
    for (int wi = 0; wi < 8; wi++) memcpy(block + off_kword(tau, wi), kbytes + 4 * wi, 4);
    for (int w = 0; w < 16; w++) memcpy(block + off_vpiece(tau, w), vbytes + 2 * w, 2);
    for (int g = 0; g < NG; g++) {
        put16(block + off_kmeta(tau, g), ks[g]);
        put16(block + off_kmeta(tau, g) + 2, kz[g]);
        put16(block + off_vmeta(tau, g), vs[g]);
        put16(block + off_vmeta(tau, g) + 2, vz[g]);
    }
}

void orc_load_token(const uint8_t *block, int tau, uint8_t *kbytes, uint8_t *vbytes,
                    uint16_t *ks, uint16_t *kz, uint16_t *vs, uint16_t *vz) {
    for (int wi = 0; wi < 8; wi++) memcpy(kbytes + 4 * wi, block + off_kword(tau, wi), 4);
    for (int w = 0; w < 16; w++) memcpy(vbytes + 2 * w, block + off_vpiece(tau, w), 2);
    for (int g = 0; g < NG; g++) {
        ks[g] = get16(block + off_kmeta(tau, g));
        kz[g] = get16(block + off_kmeta(tau, g) + 2);
        vs[g] = get16(block + off_vmeta(tau, g));
        vz[g] = get16(block + off_vmeta(tau, g) + 2);
    }
}

/* ------------------------------------------------------------------------ */
/* Attention sinks (RotateKV abstract, item (iii)).                           */
/* ------------------------------------------------------------------------ */

/* Identified sinks: the sinks are the tokens whose activations are massive.
 * act: fp32 [B][T], the activation magnitude of each of the T tokens about to
 * be appended.  Position seq_lens[b] + t becomes a sink when
 * act[b][t] >= tau while sequence b still has a free fp16 row (S rows per
 * sequence); rows are handed out in position order and recorded in
 * sink_pos[b][row], sink_count[b] = rows in use.  A sequence that the
 * append will skip (negative length, or no room for T more tokens) is
 * skipped here too. */
void orc_identify_sinks(const float *act, int B, int T, float tau, int S, int capacity,
                        const int32_t *seq_lens, int32_t *sink_pos, int32_t *sink_count) {
    for (int b = 0; b < B; b++) {
        int L0 = seq_lens[b];
        if (L0 < 0 || (int64_t)L0 + T > capacity) continue;
        for (int t = 0; t < T; t++) {
            if (act[(size_t)b * T + t] >= tau && sink_count[b] < S) {
                sink_pos[(size_t)b * S + sink_count[b]] = L0 + t;
                sink_count[b] += 1;
            }
        }
    }
}

/* The fp16 row that holds position p of sequence b, or -1 if p is stored
 * in INT2.  sink_pos == NULL: leading sinks, positions 0..S-1 are rows
 * 0..S-1.  Otherwise the identified sinks of sequence b. */
static int sink_row(int S, const int32_t *sink_pos, const int32_t *sink_count, int b, int p) {
    if (sink_pos == NULL) return p < S ? p : -1;
    for (int j = 0; j < sink_count[b] && j < S; j++)
        if (sink_pos[(size_t)b * S + j] == p) return j;
    return -1;
}

/* ------------------------------------------------------------------------ */
/* Rotate -> quantize -> append.                                              */
/* ------------------------------------------------------------------------ */

/* K, V: fp16 [B][T][Hkv][128].  R_k, R_v: fp32 [Hkv][128][128] (dense mode).
 * perm: int32 [2][Hkv][128] (FWHT mode; plane 0 keys, plane 1 values).
 * blocks: [B][Hkv][capacity/16][1536].  k_sink, v_sink: fp16 [B][Hkv][S][128].
 * seq_lens[b] (in: old length, out: old + T).  A position that is an
 * attention sink (RotateKV item (iii); sink_row above) is stored as the fp16
 * rounding of its rotated fp32 row in its sink row.  Its code slots are
 * zeroed; its meta slots too for leading sinks, while an identified sink's
 * K meta is the marker {s, z} = {0x7E00, 0} in every group (V meta zero).
 * A sequence whose new length would exceed capacity is skipped whole and
 * flags ST_CAPACITY.  Returns the status bits. */
int orc_append(const uint16_t *K, const uint16_t *V, int B, int T, int Hkv, int mode,
               const float *R_k, const float *R_v, const int32_t *perm, int capacity, int S,
               uint8_t *blocks, uint16_t *k_sink, uint16_t *v_sink, int32_t *seq_lens,
               const int32_t *sink_pos, const int32_t *sink_count) {
    int status = 0;
    const int nblk = capacity / BLK_TOK;
    for (int b = 0; b < B; b++) {
        int L0 = seq_lens[b];
        if (L0 < 0 || (int64_t)L0 + T > capacity) {
            status |= (L0 < 0) ? ST_BAD_LEN : ST_CAPACITY;
            continue;
        }
        for (int t = 0; t < T; t++) {
            int p = L0 + t;
            for (int h = 0; h < Hkv; h++) {
                const size_t src = (((size_t)b * T + t) * Hkv + h) * D;
                float kr[D], vr[D];
                orc_rotate_rows_f32(K + src, 1, mode, mode == 0 ? R_k + (size_t)h * D * D : NULL,
                                    mode == 1 ? perm + (size_t)h * D : NULL, kr);
                orc_rotate_rows_f32(V + src, 1, mode, mode == 0 ? R_v + (size_t)h * D * D : NULL,
                                    mode == 1 ? perm + ((size_t)Hkv + h) * D : NULL, vr);
                uint8_t *block = blocks + (((size_t)b * Hkv + h) * nblk + p / BLK_TOK) * BLK_BYTES;
                uint8_t kc[D], vc[D], kb[32], vb[32];
                uint16_t ks[NG], kz[NG], vs[NG], vz[NG];
                const int row = sink_row(S, sink_pos, sink_count, b, p);
                if (row >= 0) {
                    uint16_t *ksr = k_sink + (((size_t)b * Hkv + h) * S + row) * D;
                    uint16_t *vsr = v_sink + (((size_t)b * Hkv + h) * S + row) * D;
                    for (int i = 0; i < D; i++) {
                        ksr[i] = orc_f32_to_f16(kr[i]);
                        vsr[i] = orc_f32_to_f16(vr[i]);
                    }
                    memset(kb, 0, 32);
                    memset(vb, 0, 32);
                    memset(ks, 0, sizeof ks);
                    memset(kz, 0, sizeof kz);
                    memset(vs, 0, sizeof vs);
                    memset(vz, 0, sizeof vz);
                    if (sink_pos != NULL)
                        for (int g = 0; g < NG; g++) ks[g] = 0x7E00;
                } else {
                    orc_quantize_row(kr, kc, ks, kz);
                    orc_quantize_row(vr, vc, vs, vz);
                    orc_pack_row(kc, kb);
                    orc_pack_row(vc, vb);
                }
                orc_store_token(block, p % BLK_TOK, kb, vb, ks, kz, vs, vz);
            }
        }
        seq_lens[b] = L0 + T;
    }
    return status;
}

/* ------------------------------------------------------------------------ */
/* Decode attention over the packed cache (fp64).                            */
/* ------------------------------------------------------------------------ */

/* Dequantise token t of unit (b, h) into fp64 rotated K and V rows; row is
 * its fp16 sink row (sink_row), or -1 for an INT2 token. */
static void dequant_token(const uint8_t *unit_blocks, const uint16_t *ksink_u,
                          const uint16_t *vsink_u, int row, int t, double *k, double *v) {
    if (row >= 0) {
        for (int i = 0; i < D; i++) {
            k[i] = (double)orc_f16_to_f32(ksink_u[(size_t)row * D + i]);
            v[i] = (double)orc_f16_to_f32(vsink_u[(size_t)row * D + i]);
        }
        return;
    }
    const uint8_t *block = unit_blocks + (size_t)(t / BLK_TOK) * BLK_BYTES;
    uint8_t kb[32], vb[32], kc[D], vc[D];
    uint16_t ks[NG], kz[NG], vs[NG], vz[NG];
    orc_load_token(block, t % BLK_TOK, kb, vb, ks, kz, vs, vz);
    orc_unpack_row(kb, kc);
    orc_unpack_row(vb, vc);
    for (int j = 0; j < D; j++) {
        int g = j / GS;
        k[j] = (double)kc[j] * (double)orc_f16_to_f32(ks[g]) + (double)orc_f16_to_f32(kz[g]);
        v[j] = (double)vc[j] * (double)orc_f16_to_f32(vs[g]) + (double)orc_f16_to_f32(vz[g]);
    }
}

/* KVLinC's key correction adapter ("KVLinC : KV Cache Quantization with
 * Hadamard Rotation and Linear Correction", abstract: lightweight linear
 * correction adapters compensate for the errors introduced by quantized
 * keys).  The page gives no formula; the reading taken: a linear map of the
 * dequantised key in the model's (unrotated) basis, of rank r,
 *     k~ = k^ + (k^ . U) . V^T,      U, V: [128][r] (row-major, fp32),
 * applied to every INT2 key; fp16 sink keys carry no quantization error and
 * are used as stored.  U = 0 or V = 0 is the plain decode. */
static void adapt_key(const double *k_un, const float *U, const float *V, int r, double *out) {
    double kU[D];
    for (int j = 0; j < r; j++) {
        double acc = 0.0;
        for (int i = 0; i < D; i++) acc += k_un[i] * (double)U[i * r + j];
        kU[j] = acc;
    }
    for (int i = 0; i < D; i++) {
        double acc = 0.0;
        for (int j = 0; j < r; j++) acc += kU[j] * (double)V[i * r + j];
        out[i] = k_un[i] + acc;
    }
}

/* One (b, query head): q_rot = q . R_k, scores s_t = q_rot . k_t / sqrt(128)
 * over t in [0, L), softmax, o_rot = sum p_t v_t, out = o_rot . R_v^T.
 * Query head h uses KV head h / G (contiguous GQA grouping).  With an
 * adapter (U != NULL), an INT2 key is taken back to the model's basis
 * (k^ = k_rot . R_k^T), corrected (adapt_key), and scored against the
 * unrotated query: s_t = q . k~ / sqrt(128). */
static void decode_one(const uint16_t *q, int mode, const float *Rk, const float *Rv,
                       const int32_t *pk, const int32_t *pv, const uint8_t *unit_blocks,
                       const uint16_t *ksink_u, const uint16_t *vsink_u, int S,
                       const int32_t *sink_pos, const int32_t *sink_count, int b, int L,
                       const float *U, const float *V, int r, double *out) {
    double qin[D], qr[D], k[D], v[D], o[D], kun[D], kad[D];
    for (int i = 0; i < D; i++) qin[i] = (double)orc_f16_to_f32(q[i]);
    rotate_f64(qin, mode, Rk, pk, qr);
    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    const double scale = 1.0 / sqrt((double)D);
    double m = -INFINITY;
    for (int t = 0; t < L; t++) {
        const int row = sink_row(S, sink_pos, sink_count, b, t);
        dequant_token(unit_blocks, ksink_u, vsink_u, row, t, k, v);
        double acc = 0.0;
        if (U && row < 0) {
            unrotate_f64(k, mode, Rk, pk, kun);
            adapt_key(kun, U, V, r, kad);
            for (int i = 0; i < D; i++) acc += qin[i] * kad[i];
        } else {
            for (int i = 0; i < D; i++) acc += qr[i] * k[i];
        }
        s[t] = acc * scale;
        if (s[t] > m) m = s[t];
    }
    double l = 0.0;
    for (int i = 0; i < D; i++) o[i] = 0.0;
    for (int t = 0; t < L; t++) {
        double p = exp(s[t] - m);
        l += p;
        dequant_token(unit_blocks, ksink_u, vsink_u, sink_row(S, sink_pos, sink_count, b, t), t, k, v);
        for (int i = 0; i < D; i++) o[i] += p * v[i];
    }
    for (int i = 0; i < D; i++) o[i] /= l;
    unrotate_f64(o, mode, Rv, pv, out);
    free(s);
}

/* Q: fp16 [B][Hq][128].  out: fp64 [B][Hq][128].  sink_pos / sink_count:
 * identified sinks of each sequence, or NULL for leading sinks (the
 * position-to-row map is sink_row's).  Units with an invalid
 * length (L < 1 or L > capacity) get out = 0 and flag ST_BAD_LEN.
 * only_b / only_h >= 0 restrict the work to one sequence / KV head (used to
 * sample large workloads); other outputs are left untouched.
 * n_threads > 1 runs (b, query head) pairs on that many OpenMP threads. */
static int decode_all(const uint16_t *Q, int B, int Hq, int Hkv, int mode, const float *R_k,
                      const float *R_v, const int32_t *perm, int capacity, int S,
                      const uint8_t *blocks, const uint16_t *k_sink, const uint16_t *v_sink,
                      const int32_t *seq_lens, const int32_t *sink_pos,
                      const int32_t *sink_count, const float *U, const float *V, int r,
                      int only_b, int only_h, int n_threads, double *out) {
    int status = 0;
    const int G = Hq / Hkv;
    const int nblk = capacity / BLK_TOK;
    for (int b = 0; b < B; b++) {
        int L = seq_lens[b];
        if ((only_b < 0 || b == only_b) && (L < 1 || L > capacity)) status |= ST_BAD_LEN;
    }
    const int64_t npairs = (int64_t)B * Hq;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
    for (int64_t bh = 0; bh < npairs; bh++) {
        int b = (int)(bh / Hq), hq = (int)(bh % Hq), h = hq / G;
        if (only_b >= 0 && b != only_b) continue;
        if (only_h >= 0 && h != only_h) continue;
        double *o = out + (size_t)bh * D;
        int L = seq_lens[b];
        if (L < 1 || L > capacity) {
            for (int i = 0; i < D; i++) o[i] = 0.0;
            continue;
        }
        const size_t u = (size_t)b * Hkv + h;
        decode_one(Q + (size_t)bh * D, mode, mode == 0 ? R_k + (size_t)h * D * D : NULL,
                   mode == 0 ? R_v + (size_t)h * D * D : NULL,
                   mode == 1 ? perm + (size_t)h * D : NULL,
                   mode == 1 ? perm + ((size_t)Hkv + h) * D : NULL,
                   blocks + u * (size_t)nblk * BLK_BYTES,
                   S > 0 ? k_sink + u * (size_t)S * D : NULL,
                   S > 0 ? v_sink + u * (size_t)S * D : NULL, S, sink_pos, sink_count, b, L,
                   U ? U + (size_t)h * D * r : NULL, U ? V + (size_t)h * D * r : NULL, r, o);
    }
    return status;
}

int orc_decode(const uint16_t *Q, int B, int Hq, int Hkv, int mode, const float *R_k,
               const float *R_v, const int32_t *perm, int capacity, int S,
               const uint8_t *blocks, const uint16_t *k_sink, const uint16_t *v_sink,
               const int32_t *seq_lens, const int32_t *sink_pos, const int32_t *sink_count,
               int only_b, int only_h, int n_threads, double *out) {
    return decode_all(Q, B, Hq, Hkv, mode, R_k, R_v, perm, capacity, S, blocks, k_sink, v_sink,
                      seq_lens, sink_pos, sink_count, NULL, NULL, 0, only_b, only_h, n_threads,
                      out);
}

/* orc_decode with KVLinC key correction adapters U, V: fp32 [Hkv][128][r]
 * (adapt_key, per KV head). */
int orc_decode_adapter(const uint16_t *Q, int B, int Hq, int Hkv, int mode, const float *R_k,
                       const float *R_v, const int32_t *perm, int capacity, int S,
                       const uint8_t *blocks, const uint16_t *k_sink, const uint16_t *v_sink,
                       const int32_t *seq_lens, const int32_t *sink_pos,
                       const int32_t *sink_count, const float *U, const float *V, int r,
                       int n_threads, double *out) {
    return decode_all(Q, B, Hq, Hkv, mode, R_k, R_v, perm, capacity, S, blocks, k_sink, v_sink,
                      seq_lens, sink_pos, sink_count, U, V, r, -1, -1, n_threads, out);
}

/* Attention over explicit fp64 rows (no cache, no quantization), used by the
 * rotation-invariance pin: out = softmax(q . K^T / sqrt(128)) V. */
void orc_attention_f64(const double *q, const double *K, const double *V, int L, double *out) {
    const double scale = 1.0 / sqrt((double)D);
    double *s = (double *)malloc(sizeof(double) * (size_t)L);
    double m = -INFINITY, l = 0.0;
    for (int t = 0; t < L; t++) {
        double acc = 0.0;
        for (int i = 0; i < D; i++) acc += q[i] * K[(size_t)t * D + i];
        s[t] = acc * scale;
        if (s[t] > m) m = s[t];
    }
    for (int i = 0; i < D; i++) out[i] = 0.0;
    for (int t = 0; t < L; t++) {
        double p = exp(s[t] - m);
        l += p;
        for (int i = 0; i < D; i++) out[i] += p * V[(size_t)t * D + i];
    }
    for (int i = 0; i < D; i++) out[i] /= l;
    free(s);
}

/* Array forms of the binary16 conversions (one call per array). */
void orc_f32_to_f16_array(const float *x, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; i++) out[i] = orc_f32_to_f16(x[i]);
}

void orc_f16_to_f32_array(const uint16_t *x, int64_t n, float *out) {
    for (int64_t i = 0; i < n; i++) out[i] = orc_f16_to_f32(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Pre-RoPE grouped-head rotation (RotateKV abstract, item (ii)).             */
/* ------------------------------------------------------------------------ */
/* Keys are rotated before RoPE, and one rotation spans the keys of a group
 * of gh consecutive KV heads: the concatenation x (n = 128*gh channels) is
 * reordered, y[i] = x[perm[i]] (perm a permutation of 0..n-1), and
 * x_rot = FWHT_n(y)/sqrt(n).  Each head's 128-channel slice of x_rot is
 * quantized and stored in that head's cache unit.  At decode time the key
 * of position t is the inverse rotation of the dequantised group row, then
 * RoPE at position t.  Values are rotated per head, as in FWHT mode.
 *
 * RoPE (rotate-half pairing): channel c < 64 pairs with c + 64, with
 * frequency theta_c = base^(-2c/128) and angle t * theta_c:
 *   out[c]      = x[c] cos(a) - x[c+64] sin(a)
 *   out[c + 64] = x[c+64] cos(a) + x[c] sin(a). */

void orc_rope_f64(double *x, int64_t t, double base) {
    for (int c = 0; c < D / 2; c++) {
        const double th = pow(base, -2.0 * (double)c / (double)D);
        const double a = (double)t * th;
        const double cs = cos(a), sn = sin(a);
        const double x0 = x[c], x1 = x[c + D / 2];
        x[c] = x0 * cs - x1 * sn;
        x[c + D / 2] = x1 * cs + x0 * sn;
    }
}

/* x (n channels) -> FWHT_n(x[perm]) / sqrt(n). */
void orc_rotate_group_f64(const double *x, int n, const int32_t *perm, double *out) {
    for (int i = 0; i < n; i++) out[i] = x[perm[i]];
    orc_fwht_f64(out, n);
    const double sc = 1.0 / sqrt((double)n);
    for (int i = 0; i < n; i++) out[i] *= sc;
}

/* The inverse: y = FWHT_n(o) / sqrt(n), out[perm[i]] = y[i]. */
void orc_unrotate_group_f64(const double *o, int n, const int32_t *perm, double *out) {
    double *y = (double *)malloc(sizeof(double) * (size_t)n);
    for (int i = 0; i < n; i++) y[i] = o[i];
    orc_fwht_f64(y, n);
    const double sc = 1.0 / sqrt((double)n);
    for (int i = 0; i < n; i++) out[perm[i]] = y[i] * sc;
    free(y);
}

/* Pre-RoPE append.  K (pre-RoPE), V: fp16 [B][T][Hkv][128]; gh divides Hkv;
 * perm int32 [2][Hkv*128]: plane 0 holds Hkv/gh key permutations of n =
 * 128*gh entries each (group q at perm + q*n), plane 1 one value permutation
 * of 128 entries per head.  Sinks (RotateKV item (iii); sink_row above): the
 * sink row keeps the key as given (pre-RoPE, not rotated: it is never
 * quantized, and RoPE is applied at decode time) and the rotated value in
 * fp16; the INT2 slot is zeroed, with the K-meta marker for identified
 * sinks.  Returns the status bits; seq_lens advance by T for every sequence
 * that fits. */
int orc_append_prerope(const uint16_t *K, const uint16_t *V, int B, int T, int Hkv, int gh,
                       const int32_t *perm, int capacity, int S, uint8_t *blocks,
                       uint16_t *k_sink, uint16_t *v_sink, int32_t *seq_lens,
                       const int32_t *sink_pos, const int32_t *sink_count) {
    int status = 0;
    const int nblk = capacity / BLK_TOK;
    const int n = D * gh;
    double *xg = (double *)malloc(sizeof(double) * (size_t)n);
    double *xr = (double *)malloc(sizeof(double) * (size_t)n);
    for (int b = 0; b < B; b++) {
        const int L0 = seq_lens[b];
        if (L0 < 0 || (int64_t)L0 + T > capacity) {
            status |= (L0 < 0) ? ST_BAD_LEN : ST_CAPACITY;
            continue;
        }
        for (int t = 0; t < T; t++) {
            const int p = L0 + t;
            for (int q = 0; q < Hkv / gh; q++) {
                for (int j = 0; j < gh; j++)
                    for (int i = 0; i < D; i++)
                        xg[j * D + i] = (double)orc_f16_to_f32(
                            K[(((size_t)b * T + t) * Hkv + q * gh + j) * D + i]);
                orc_rotate_group_f64(xg, n, perm + (size_t)q * n, xr);
                const int row = sink_row(S, sink_pos, sink_count, b, p);
                for (int j = 0; j < gh; j++) {
                    const int h = q * gh + j;
                    float kr[D], vr[D];
                    for (int i = 0; i < D; i++) kr[i] = (float)xr[j * D + i];
                    orc_rotate_rows_f32(V + (((size_t)b * T + t) * Hkv + h) * D, 1, 1, NULL,
                                        perm + ((size_t)Hkv + h) * D, vr);
                    uint8_t kc[D], vc[D], kb[32], vb[32];
                    uint16_t ks[NG], kz[NG], vs[NG], vz[NG];
                    if (row >= 0) {
                        const uint16_t *kin = K + (((size_t)b * T + t) * Hkv + h) * D;
                        uint16_t *ksr = k_sink + (((size_t)b * Hkv + h) * S + row) * D;
                        uint16_t *vsr = v_sink + (((size_t)b * Hkv + h) * S + row) * D;
                        for (int i = 0; i < D; i++) {
                            ksr[i] = kin[i];
                            vsr[i] = orc_f32_to_f16(vr[i]);
                        }
                        memset(kb, 0, 32);
                        memset(vb, 0, 32);
                        memset(ks, 0, sizeof ks);
                        memset(kz, 0, sizeof kz);
                        memset(vs, 0, sizeof vs);
                        memset(vz, 0, sizeof vz);
                        if (sink_pos != NULL)
                            for (int g = 0; g < NG; g++) ks[g] = 0x7E00;
                    } else {
                        orc_quantize_row(kr, kc, ks, kz);
                        orc_quantize_row(vr, vc, vs, vz);
                        orc_pack_row(kc, kb);
                        orc_pack_row(vc, vb);
                    }
                    uint8_t *block =
                        blocks + (((size_t)b * Hkv + h) * nblk + p / BLK_TOK) * BLK_BYTES;
                    orc_store_token(block, p % BLK_TOK, kb, vb, ks, kz, vs, vz);
                }
            }
        }
        seq_lens[b] = L0 + T;
    }
    free(xg);
    free(xr);
    return status;
}

/* Pre-RoPE decode.  Q: fp16 [B][Hq][128] post-RoPE queries (query head hq
 * reads KV head hq / G).  For every position t < L: the dequantised rotated
 * key rows of the gh heads of the group, inversely rotated, the head's slice
 * taken and RoPE'd at position t (a sink: its stored pre-RoPE key RoPE'd);
 * s_t = q . k_t / sqrt(128); softmax; the values as in FWHT mode:
 * o_rot = sum p_t v_t, out = FWHT(o_rot)/sqrt(128) scattered through the
 * head's value permutation.  Output fp64 [B][Hq][128]; invalid lengths give
 * zeros and ST_BAD_LEN. */
int orc_decode_prerope(const uint16_t *Q, int B, int Hq, int Hkv, int gh, const int32_t *perm,
                       double rope_base, int capacity, int S, const uint8_t *blocks,
                       const uint16_t *k_sink, const uint16_t *v_sink, const int32_t *seq_lens,
                       const int32_t *sink_pos, const int32_t *sink_count, int only_b,
                       int only_h, int n_threads, double *out) {
    int status = 0;
    const int G = Hq / Hkv;
    const int nblk = capacity / BLK_TOK;
    const int n = D * gh;
    for (int b = 0; b < B; b++) {
        const int L = seq_lens[b];
        if ((only_b < 0 || b == only_b) && (L < 1 || L > capacity)) status |= ST_BAD_LEN;
    }
    const int64_t npairs = (int64_t)B * Hq;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
    for (int64_t bh = 0; bh < npairs; bh++) {
        const int b = (int)(bh / Hq), hq = (int)(bh % Hq), h = hq / G;
        const int q = h / gh, j = h % gh;
        if (only_b >= 0 && b != only_b) continue;
        if (only_h >= 0 && h != only_h) continue;
        double *o = out + (size_t)bh * D;
        const int L = seq_lens[b];
        if (L < 1 || L > capacity) {
            for (int i = 0; i < D; i++) o[i] = 0.0;
            continue;
        }
        double qv[D], k[D], v[D], orot[D];
        for (int i = 0; i < D; i++) qv[i] = (double)orc_f16_to_f32(Q[(size_t)bh * D + i]);
        double *kg = (double *)malloc(sizeof(double) * (size_t)n);
        double *ku = (double *)malloc(sizeof(double) * (size_t)n);
        double *s = (double *)malloc(sizeof(double) * (size_t)L);
        const double scale = 1.0 / sqrt((double)D);
        double m = -INFINITY;
        const size_t uh = (size_t)b * Hkv + h;
        for (int t = 0; t < L; t++) {
            const int row = sink_row(S, sink_pos, sink_count, b, t);
            if (row >= 0) {
                for (int i = 0; i < D; i++)
                    k[i] = (double)orc_f16_to_f32(k_sink[(uh * S + row) * D + i]);
            } else {
                for (int jj = 0; jj < gh; jj++) {
                    const size_t u = (size_t)b * Hkv + q * gh + jj;
                    dequant_token(blocks + u * (size_t)nblk * BLK_BYTES, NULL, NULL, -1, t, k, v);
                    for (int i = 0; i < D; i++) kg[jj * D + i] = k[i];
                }
                orc_unrotate_group_f64(kg, n, perm + (size_t)q * n, ku);
                for (int i = 0; i < D; i++) k[i] = ku[j * D + i];
            }
            orc_rope_f64(k, t, rope_base);
            double acc = 0.0;
            for (int i = 0; i < D; i++) acc += qv[i] * k[i];
            s[t] = acc * scale;
            if (s[t] > m) m = s[t];
        }
        double l = 0.0;
        for (int i = 0; i < D; i++) orot[i] = 0.0;
        for (int t = 0; t < L; t++) {
            const double p = exp(s[t] - m);
            l += p;
            dequant_token(blocks + uh * (size_t)nblk * BLK_BYTES,
                          S > 0 ? k_sink + uh * (size_t)S * D : NULL,
                          S > 0 ? v_sink + uh * (size_t)S * D : NULL,
                          sink_row(S, sink_pos, sink_count, b, t), t, k, v);
            for (int i = 0; i < D; i++) orot[i] += p * v[i];
        }
        for (int i = 0; i < D; i++) orot[i] /= l;
        unrotate_f64(orot, 1, NULL, perm + ((size_t)Hkv + h) * D, o);
        free(kg);
        free(ku);
        free(s);
    }
    return status;
}
