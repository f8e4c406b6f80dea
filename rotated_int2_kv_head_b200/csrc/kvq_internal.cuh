// Device-side helpers shared by the libkvq kernels: cache-block offsets, the
// exact INT2 group quantizer, fp16 helpers, and mbarrier / bulk-copy PTX.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvq.h"

namespace kvq {

constexpr int D = 128;          // head_dim
constexpr int GS = 32;          // quantization group (elements of head_dim)
constexpr int NG = D / GS;      // groups per row
constexpr int BLK_TOK = 16;     // tokens per cache block
constexpr int BLK_BYTES = 1536; // bytes per cache block (96 per token)
constexpr int OFF_VC = 512, OFF_KM = 1024, OFF_VM = 1280;
constexpr int MAX_SINK = 64;

// ---- cache block offsets (format documented in include/kvq.h) ---------------------
// tau = token in block.  K code word wi = logical bytes 4wi..4wi+3.
__device__ __forceinline__ int off_kword(int tau, int wi) {
    const int r = tau & 7, th = tau >> 3;
    return 16 * (4 * r + (wi & 3)) + 4 * (2 * th + (wi >> 2));
}
// V code piece w = logical bytes 2w, 2w+1 of the token.
__device__ __forceinline__ int off_vpiece(int tau, int w) {
    const int q = tau >> 1, side = tau & 1;
    return OFF_VC + 16 * (4 * (w & 7) + (q & 3)) + 4 * (2 * (q >> 2) + (w >> 3)) + 2 * side;
}
__device__ __forceinline__ int off_kmeta(int tau, int g) {
    const int r = tau & 7, th = tau >> 3;
    return OFF_KM + 8 * (4 * r + g) + 4 * th;
}
__device__ __forceinline__ int off_vmeta(int tau, int g) {
    const int r = tau & 7, th = tau >> 3;
    return OFF_VM + 8 * (4 * r + g) + 4 * th;
}

__device__ __forceinline__ void set_status(int32_t *status, int bits) {
    if (status) atomicOr(reinterpret_cast<int *>(status), bits);
}

// ---- exact INT2 group quantizer -----------------------------------------------------
// One warp holds one 128-element rotated fp32 row, lane l holding elements
// 4l..4l+3 (so lanes 8g..8g+7 hold group g).  Arithmetic is the documented
// IEEE fp32 sequence with explicit round-to-nearest intrinsics (no
// contraction), so it matches the reference quantizer bit for bit:
//   s = fp16((max-min)/3), z = fp16(min), inv = s ? 1/s : 0,
//   c = clamp(rint((x - z) * inv), 0, 3).
// Returns, in every lane, the logical code word for bytes 4*(l%8)..+3 (the
// byte e carries element e of each group at bits 2g) and the lane's group
// scale/zero as fp16 bits.
struct QuantWord {
    uint32_t word;
    uint16_t s, z;
};

// Three-input fp32 min / max (one instruction each).
__device__ __forceinline__ float fmin3(float a, float b, float c) {
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Per element the code is formed without a float-to-int conversion: clamp t
// to [0, 3] first (clamping then rounding equals rounding then clamping on
// that interval), then add 1.5 * 2^23, after which fp32 round-to-nearest-
// even leaves rint(t) in the low mantissa bits (bit pattern 0x4B400000 + c).
// The four patterns are added into the word at their codes' places and the
// constant terms taken out once.  1/s is the correctly rounded reciprocal
// (__frcp_rn), the same value as the IEEE division 1/s.
__device__ __forceinline__ QuantWord quantize_row_warp(const float v[4]) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 3;
    float mn = fminf(fmin3(v[0], v[1], v[2]), v[3]);
    float mx = fmaxf(fmax3(v[0], v[1], v[2]), v[3]);
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    const float r = __fsub_rn(mx, mn);
    const float sf = __fdiv_rn(r, 3.0f);
    const __half s = __float2half_rn(__fadd_rn(sf, 0.0f));   // zero stored as +0
    const __half z = __float2half_rn(__fadd_rn(mn, 0.0f));
    const float sF = __half2float(s), zF = __half2float(z);
    const float inv = (sF == 0.0f) ? 0.0f : __frcp_rn(sF);
    constexpr float MAGIC = 12582912.0f;                     // 1.5 * 2^23
    constexpr uint32_t MAGIC_BITS = 0x4B400000u;
    uint32_t bits = 0;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        float t = __fmul_rn(__fsub_rn(v[k], zF), inv);
        t = fminf(fmaxf(t, 0.0f), 3.0f);
        bits += __float_as_uint(__fadd_rn(t, MAGIC)) << (8 * k + 2 * g);
    }
    bits -= (MAGIC_BITS << (2 * g)) + (MAGIC_BITS << (8 + 2 * g)) + (MAGIC_BITS << (16 + 2 * g)) +
            (MAGIC_BITS << (24 + 2 * g));
    bits |= __shfl_xor_sync(0xffffffffu, bits, 8);
    bits |= __shfl_xor_sync(0xffffffffu, bits, 16);
    QuantWord q;
    q.word = bits;
    q.s = __half_as_ushort(s);
    q.z = __half_as_ushort(z);
    return q;
}

// Two fp32 values in one 64-bit register, for sm_100's paired fp32
// sub / mul: each lane is rounded to nearest even exactly as the
// scalar instruction rounds it.  Unlike a scalar add.rn / mul.rn, a paired
// product followed by a paired sum may be contracted into one fused
// multiply-add by the assembler (one rounding instead of two; seen on
// sm_100a), so where the exact two-step result matters a paired product
// only ever feeds a scalar .rn operation.
__device__ __forceinline__ uint64_t f2_make(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t x, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x));
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// v[e] *= c for the 32 values of a group, one rounding per value (scalar
// mul.rn, never contracted with the subtraction that follows it in the
// quantizer).
__device__ __forceinline__ void scale_group(float (&v)[32], float c) {
#pragma unroll
    for (int e = 0; e < 32; e++) v[e] = __fmul_rn(v[e], c);
}

// One thread quantizes one group g of one row: v holds the group's 32
// rotated values.  The codes are added into the 8 logical code words of the
// row (word w = bytes 4w..4w+3; element e of the group at byte e, bits 2g)
// with the magic-constant rounding of quantize_row_warp (each pattern added
// at its code's place with one integer multiply-add, the codes' bits never
// overlapping, the constant terms taken out once per word); min and max by
// three-input min/max trees.  Returns the meta word {s, z}.  Same
// arithmetic as quantize_row_warp, bit for bit.
__device__ __forceinline__ uint32_t quantize_group_thread(const float (&v)[32], int g,
                                                          uint32_t (&words)[8]) {
    // min and max of the 32 values with three-input min/max: 32 -> 12 -> 4 -> 1
    float mn[12], mx[12];
#pragma unroll
    for (int e = 0; e < 10; e++) {
        mn[e] = fmin3(v[3 * e], v[3 * e + 1], v[3 * e + 2]);
        mx[e] = fmax3(v[3 * e], v[3 * e + 1], v[3 * e + 2]);
    }
    mn[10] = v[30], mn[11] = v[31], mx[10] = v[30], mx[11] = v[31];
#pragma unroll
    for (int e = 0; e < 4; e++) {
        mn[e] = fmin3(mn[3 * e], mn[3 * e + 1], mn[3 * e + 2]);
        mx[e] = fmax3(mx[3 * e], mx[3 * e + 1], mx[3 * e + 2]);
    }
    mn[0] = fminf(fmin3(mn[0], mn[1], mn[2]), mn[3]);
    mx[0] = fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
    const float r = __fsub_rn(mx[0], mn[0]);
    const float sf = __fdiv_rn(r, 3.0f);
    const __half s = __float2half_rn(__fadd_rn(sf, 0.0f));   // zero stored as +0
    const __half z = __float2half_rn(__fadd_rn(mn[0], 0.0f));
    const float sF = __half2float(s), zF = __half2float(z);
    const float inv = (sF == 0.0f) ? 0.0f : __frcp_rn(sF);   // = the IEEE quotient 1/s
    constexpr float MAGIC = 12582912.0f;                     // 1.5 * 2^23
    constexpr uint32_t MAGIC_BITS = 0x4B400000u;
    // sum_j (MAGIC_BITS << (8j + 2g)) (mod 2^32), taken out of every word
    const uint32_t magic_sum = (MAGIC_BITS << (2 * g)) + (MAGIC_BITS << (8 + 2 * g)) +
                               (MAGIC_BITS << (16 + 2 * g)) + (MAGIC_BITS << (24 + 2 * g));
    // Every t = (x - z) * inv of the group lies in [t(min), t(max)]: the
    // rounded difference and its rounded product with inv >= 0 are monotone
    // in x.  When that interval lies in [-0.5, 3.5), rounding alone already
    // gives every code the clamped value (t in [-0.5, 0) rounds to 0, the
    // tie -0.5 to even 0; t in (3, 3.5) rounds to 3), so the clamp is
    // skipped and x - z and its product with inv run two elements per
    // instruction (the magic-constant sum stays a scalar add.rn, which is
    // never fused with the product).  A NaN or infinite bound fails the
    // test and takes the clamped path.
    const float tlo = __fmul_rn(__fsub_rn(mn[0], zF), inv);
    const float thi = __fmul_rn(__fsub_rn(mx[0], zF), inv);
    if (tlo >= -0.5f && thi < 3.5f) {
        const uint64_t z2 = f2_make(zF, zF), i2 = f2_make(inv, inv);
#pragma unroll
        for (int w = 0; w < 8; w++) {
            uint32_t acc = words[w];
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
                const int e = 4 * w + j;
                float a, b;
                f2_split(f2_mul(f2_sub(f2_make(v[e], v[e + 1]), z2), i2), a, b);
                acc += __float_as_uint(__fadd_rn(a, MAGIC)) << (8 * j + 2 * g);
                acc += __float_as_uint(__fadd_rn(b, MAGIC)) << (8 * (j + 1) + 2 * g);
            }
            words[w] = acc - magic_sum;
        }
    } else {
#pragma unroll
        for (int w = 0; w < 8; w++) {
            uint32_t acc = words[w];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int e = 4 * w + j;
                float t = __fmul_rn(__fsub_rn(v[e], zF), inv);
                t = fminf(fmaxf(t, 0.0f), 3.0f);
                acc += __float_as_uint(__fadd_rn(t, MAGIC)) << (8 * j + 2 * g);
            }
            words[w] = acc - magic_sum;
        }
    }
    return (uint32_t)__half_as_ushort(s) | ((uint32_t)__half_as_ushort(z) << 16);
}

// Store one token of one kind (0 = K, 1 = V) into its block, from the warp
// layout of quantize_row_warp.  Lanes 0..7 write the code word l, lanes 8g
// write group g's metadata.
__device__ __forceinline__ void store_token_warp(uint8_t *block, int tau, int kind,
                                                 const QuantWord &q) {
    const int lane = threadIdx.x & 31;
    if (lane < 8) {
        if (kind == 0) {
            *reinterpret_cast<uint32_t *>(block + off_kword(tau, lane)) = q.word;
        } else {
            *reinterpret_cast<uint16_t *>(block + off_vpiece(tau, 2 * lane)) =
                (uint16_t)(q.word & 0xffffu);
            *reinterpret_cast<uint16_t *>(block + off_vpiece(tau, 2 * lane + 1)) =
                (uint16_t)(q.word >> 16);
        }
    }
    if ((lane & 7) == 0) {
        const int g = lane >> 3;
        *reinterpret_cast<uint32_t *>(block + (kind == 0 ? off_kmeta(tau, g) : off_vmeta(tau, g))) =
            (uint32_t)q.s | ((uint32_t)q.z << 16);
    }
}

// Zero one token's slots of one kind (sink positions).
__device__ __forceinline__ void zero_token_warp(uint8_t *block, int tau, int kind) {
    QuantWord q;
    q.word = 0;
    q.s = 0;
    q.z = 0;
    store_token_warp(block, tau, kind, q);
}

// ---- warp FWHT of a 128-vector held as 4 consecutive elements per lane -------------
// Sylvester order; butterflies (a, b) -> (a + b, a - b) at every stride.
// The cross-lane butterflies are one fma with a per-lane sign, o + sgn*v
// (sgn = -1 in the upper lane of a pair): it rounds exactly like o - v or
// v + o.
__device__ __forceinline__ void fwht128_warp(float v[4]) {
    const int lane = threadIdx.x & 31;
    float a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
    v[0] = a0 + a2;
    v[2] = a0 - a2;
    v[1] = a1 + a3;
    v[3] = a1 - a3;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const float sgn = (lane & m) ? -1.f : 1.f;
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const float o = __shfl_xor_sync(0xffffffffu, v[k], m);
            v[k] = fmaf(sgn, v[k], o);
        }
    }
}

// ---- mbarrier and bulk-copy (TMA, non-tensor) PTX wrappers ---------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    // The suspend-time hint lets the waiting thread sleep in hardware until
    // the phase completes (or ~20 us pass) instead of spinning on the issue
    // slots its SM-subpartition shares with working warps.
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}

// Bounded wait: gives up after `limit` polls (each may suspend up to the
// hint above, so the bound is about two seconds) and reports false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint32_t limit = (1u << 17)) {
    for (uint32_t i = 0; i < limit; i++)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// After a bounded wait has given up: wait, with the same bound, for the
// stages [from, issued) of a ring of ns slots (stage j fills slot j % ns,
// phase j / ns) to land, so that no bulk copy still targets this CTA's
// shared memory when it returns.  A stage whose phase is already complete
// (or that was closed by a plain arrive) passes at once.  Returns the number
// of stages that did not land within the bound (0 unless a copy itself is
// lost); the caller has already set KVQ_DEV_TIMEOUT.
__device__ __forceinline__ int drain_ring(uint64_t *full, int ns, int from, int issued) {
    int lost = 0;
    for (int j = from; j < issued; j++)
        if (!mbar_wait_bounded(&full[j % ns], (uint32_t)(j / ns) & 1u)) ++lost;
    return lost;
}

// 1-D bulk copy global -> shared, completion reported on `bar` as tx bytes.
// Both addresses 16-B aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ---- tensor-core MMA (m16n8k16, fp16 in, fp32 accumulate) ------------------------------
__device__ __forceinline__ void mma16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// m16n8k32 integer MMA: u8 A (codes) x s8 B (quantised query), s32 accumulate.
__device__ __forceinline__ void imma16832(int d[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same product into a fresh accumulator (C = 0, no zero-fill of d).
__device__ __forceinline__ void imma16832_zc(int d[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// 2^x by the SFU's ex2.approx (max relative error about 2^-22; results
// below 2^-126 flush to 0, which a softmax weight may do).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ float2 unpack_half2(uint32_t u) {
    const __half2 h = *reinterpret_cast<const __half2 *>(&u);
    return __half22float2(h);
}

// ---- programmatic dependent launch ---------------------------------------------------------
// Every kernel is launched with programmatic stream serialisation, so it may
// start while the previous kernel in the stream drains.  Each kernel calls
// pdl_wait() (the previous grid has completed and its writes are visible)
// before it reads anything the previous kernel may write, and only then
// pdl_trigger() to let the next kernel launch.  Hence when a kernel starts,
// every grid before its predecessor has completed; work placed before
// pdl_wait() touches only data no earlier kernel of the chain writes.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---- host launchers (defined in kvq_append.cu / kvq_decode.cu) ---------------------------
cudaError_t launch_append_small(const uint16_t *K, const uint16_t *V, int T, int mode,
                                const float *R_k, const float *R_v, const int32_t *perm,
                                const kvq_cache_desc &cd, int32_t *seq_lens,
                                cudaStream_t st);
cudaError_t launch_debug_rotate_small(const uint16_t *X, int N, int mode, const float *R,
                                      const int32_t *perm, float *out, cudaStream_t st);
// Whether an append of T rows per sequence over B sequences (16-byte aligned
// K and V) runs its rotation on the tensor cores (the size rule is beside
// the kernel).
bool append_tc_eligible(int mode, const uint16_t *K, const uint16_t *V, int T, int B);
cudaError_t launch_append_tc(const uint16_t *K, const uint16_t *V, int T, int mode,
                             const float *R_k, const float *R_v, const int32_t *perm,
                             const kvq_cache_desc &cd, int32_t *seq_lens, cudaStream_t st);
cudaError_t launch_debug_rotate_tc(const uint16_t *X, int N, int mode, const float *R,
                                   const int32_t *perm, float *out, cudaStream_t st);
cudaError_t launch_debug_quantize(const float *X, int N, uint8_t *codes, uint16_t *meta,
                                  cudaStream_t st);
cudaError_t launch_debug_wait_timeout(const uint8_t *src, uint32_t poll_limit, int32_t *status,
                                      int32_t *result, cudaStream_t st);
cudaError_t launch_identify_sinks(const float *act, int T, float tau, const kvq_cache_desc &cd,
                                  const int32_t *seq_lens, cudaStream_t st);
// pre-RoPE grouped-head key rotation (kvq_append.cu / kvq_prerope.cu)
cudaError_t launch_append_prerope(const uint16_t *K, const uint16_t *V, int T, int gh,
                                  const int32_t *perm, const kvq_cache_desc &cd,
                                  int32_t *seq_lens, cudaStream_t st);
cudaError_t launch_debug_rotate_group(const uint16_t *X, int N, int gh, const int32_t *perm,
                                     float *out, cudaStream_t st);
size_t prerope_ws_bytes(int B, int Hq, int Hkv, int gh, int max_ctx, int sms);
cudaError_t launch_decode_prerope(const uint16_t *Q, int Hq, const kvq_cache_desc &cd, int gh,
                                  const int32_t *perm, float rope_base, const int32_t *seq_lens,
                                  int max_ctx, int sms, void *ws, uint16_t *out, cudaStream_t st);
// KVLinC key correction adapter of a decode: U, V fp32 [Hkv][128][r], or
// none (U = nullptr).
struct KeyAdapter {
    const float *U = nullptr, *V = nullptr;
    int r = 0;
};
cudaError_t launch_decode(const uint16_t *Q, int Hq, const kvq_cache_desc &cd, int mode,
                          const float *R_k, const float *R_v, const int32_t *perm,
                          const int32_t *seq_lens, int C, void *ws, uint16_t *out,
                          cudaStream_t st, cudaEvent_t ev_begin, cudaEvent_t ev_end, int qlen,
                          int out_rotated, const KeyAdapter &ad = KeyAdapter());

// Decode workspace: prepared queries and split partials.
struct WsLayout {
    size_t qprep, part, total;
};
WsLayout ws_layout(int B, int Hq, int Hkv, int C);


// ---- append destination and completion (shared by the append kernels) ---------------
// Where a rotated row goes: into the packed cache, or out as fp32 (tests).
struct CacheDst {
    uint8_t *blocks;
    uint16_t *k_sink, *v_sink;
    int32_t *seq_lens;
    int32_t *status;          // [0] error bits, [1] CTA completion counter
    int B, T, Hkv, capacity, S, nblk;
    const int32_t *table;     // paged cache: [B][nblk] pool block per logical block, else null
    int num_blocks;           // paged: pool blocks
    int32_t *sink_pos;        // identified sinks: [B][S] ascending positions, else null
    int32_t *sink_count;      // identified sinks: [B] rows in use
};

// The append destination of cache `cd`.
inline CacheDst cache_dst(const kvq_cache_desc &cd, int32_t *seq_lens, int T) {
    CacheDst c;
    c.blocks = static_cast<uint8_t *>(cd.blocks);
    c.table = cd.block_table;
    c.num_blocks = cd.num_blocks;
    c.k_sink = cd.k_sink;
    c.v_sink = cd.v_sink;
    c.seq_lens = seq_lens;
    c.status = cd.status;
    c.B = cd.B;
    c.T = T;
    c.Hkv = cd.Hkv;
    c.capacity = cd.capacity;
    c.S = cd.sink_fp16;
    c.nblk = cd.capacity / BLK_TOK;
    c.sink_pos = cd.sink_pos;
    c.sink_count = cd.sink_count;
    return c;
}

// K meta word {s, z} of an identified sink's INT2 slot in every group: s is
// the fp16 quiet NaN 0x7E00, z = 0.  Any score computed from it is NaN,
// which the decode turns into -inf.
constexpr uint32_t SINK_KMETA_MARK = 0x7E00u;

// fp16 sink row of position p of sequence b, or -1 if p is stored in INT2.
// Leading sinks: positions 0..S-1 are rows 0..S-1.  Identified sinks: the
// index of p in the sequence's ascending list; `last` is the list's last
// entry (or -1 for an empty list), which almost every position lies past.
__device__ __forceinline__ int sink_row_after(const CacheDst &c, int b, int p, int n, int last) {
    if (!c.sink_pos) return p < c.S ? p : -1;
    if (p > last) return -1;
    const int32_t *sp = c.sink_pos + (size_t)b * c.S;
    int lo = 0, hi = n - 1;                      // first entry >= p (one exists: p <= last)
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (sp[mid] < p) lo = mid + 1; else hi = mid;
    }
    return sp[lo] == p ? lo : -1;
}
// Rows in use and last listed position of sequence b (identified sinks).
__device__ __forceinline__ void sink_list_end(const CacheDst &c, int b, int &n, int &last) {
    n = 0;
    last = -1;
    if (!c.sink_pos) return;
    n = min(max(c.sink_count[b], 0), c.S);
    if (n > 0) last = c.sink_pos[(size_t)b * c.S + n - 1];
}
__device__ __forceinline__ int sink_row(const CacheDst &c, int b, int p) {
    int n, last;
    sink_list_end(c, b, n, last);
    return sink_row_after(c, b, p, n, last);
}

// Index (in 1536-byte blocks from `blocks`) of KV head h of logical block lb
// of sequence b; -1 for a paged entry outside the pool.
__device__ __forceinline__ long long cache_block_index(const int32_t *table, int num_blocks, int nblk,
                                                       int Hkv, int b, int h, int lb) {
    if (!table) return ((long long)b * Hkv + h) * nblk + lb;
    const int n = table[(size_t)b * nblk + lb];
    if (n < 0 || n >= num_blocks) return -1;
    return (long long)n * Hkv + h;
}

// Called by every CTA of an append kernel after its last read of seq_lens
// and its last write: the CTA that completes last bumps the lengths and
// resets the counter for the next append.
static __device__ void append_done(const CacheDst &c) {
    __shared__ int last;
    // Ordering: every thread of this CTA has read seq_lens (and used the
    // value) before the barrier, nothing writes seq_lens during the kernel,
    // and the next kernel sees the bump once this one completes, so no
    // memory fence is needed around the counter.
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned total = gridDim.x * gridDim.y * gridDim.z;
        const unsigned prev = atomicAdd(reinterpret_cast<unsigned *>(c.status + 1), 1u);
        last = (prev == total - 1);
    }
    __syncthreads();
    if (last) {
        for (int b = threadIdx.x; b < c.B; b += blockDim.x) {
            const int L0 = c.seq_lens[b];
            if (L0 >= 0 && (long long)L0 + c.T <= c.capacity) c.seq_lens[b] = L0 + c.T;
        }
        if (threadIdx.x == 0) atomicExch(reinterpret_cast<unsigned *>(c.status + 1), 0u);
    }
}

// The same completion count in two halves, for kernels whose threads read
// seq_lens only at their start: append_claim right after the last read (the
// atomic's round trip then overlaps the CTA's work), append_finish at the
// end.  The last CTA to claim bumps the lengths when it finishes: every
// other CTA has read them by then.
__device__ __forceinline__ unsigned append_claim(const CacheDst &c) {
    __syncthreads();
    unsigned prev = 0u;
    if (threadIdx.x == 0) prev = atomicAdd(reinterpret_cast<unsigned *>(c.status + 1), 1u);
    return prev;   // meaningful in thread 0
}
static __device__ void append_finish(const CacheDst &c, unsigned prev) {
    __shared__ int last;
    if (threadIdx.x == 0) last = (prev == gridDim.x * gridDim.y * gridDim.z - 1);
    __syncthreads();
    if (last) {
        for (int b = threadIdx.x; b < c.B; b += blockDim.x) {
            const int L0 = c.seq_lens[b];
            if (L0 >= 0 && (long long)L0 + c.T <= c.capacity) c.seq_lens[b] = L0 + c.T;
        }
        if (threadIdx.x == 0) atomicExch(reinterpret_cast<unsigned *>(c.status + 1), 0u);
    }
}

// Reads seq_lens[b] and checks capacity; returns -1 (and flags) if the
// sequence must be skipped.
__device__ __forceinline__ int start_len(const CacheDst &c, int b) {
    const int L0 = c.seq_lens[b];
    if (L0 < 0) {
        if (threadIdx.x == 0) set_status(c.status, KVQ_DEV_BAD_LEN);
        return -1;
    }
    if ((long long)L0 + c.T > c.capacity) {
        if (threadIdx.x == 0) set_status(c.status, KVQ_DEV_CAPACITY);
        return -1;
    }
    return L0;
}

// Per-thread variant: every caller gets L0 (or -1); only callers with
// `report` set flag the status.
__device__ __forceinline__ int start_len_thread(const CacheDst &c, int b, bool report) {
    const int L0 = c.seq_lens[b];
    if (L0 < 0) {
        if (report) set_status(c.status, KVQ_DEV_BAD_LEN);
        return -1;
    }
    if ((long long)L0 + c.T > c.capacity) {
        if (report) set_status(c.status, KVQ_DEV_CAPACITY);
        return -1;
    }
    return L0;
}

}  // namespace kvq
