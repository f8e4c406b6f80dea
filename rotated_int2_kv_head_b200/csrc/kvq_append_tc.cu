// Dense rotate -> quantize -> append on the 5th-generation tensor cores.
//
// The rotation of every appended row, x_rot = x . R for the row's KV head
// ("Output-Aware Rotation for INT2 KV-Cache Quantization", section "Key
// Details": an orthogonal rotation per head, applied before INT2
// quantization), is a dense contraction: for a bulk append (prefill) it is a
// [T x 128] . [128 x 128] product per (sequence, head, K|V).  Here it runs on
// tcgen05 with the accumulator in tensor memory:
//
//   * R (fp32) is split into two fp16 matrices, R = R_hi + R_lo with
//     R_hi = fp16(R) and R_lo = fp16(R - R_hi); x is fp16, so
//     x . R_hi + x . R_lo carries about 22 bits of R and accumulates in fp32.
//   * warp 0 streams 128-row tiles of x with 3-D TMA copies (128-byte
//     swizzle, the layout the MMA reads) into a 3-stage ring;
//   * warp 1 owns all 512 TMEM columns (four 128x128 fp32 accumulators) and
//     issues, per tile, 16 tcgen05.mma (hi and lo, K = 128 in steps of 16);
//   * warps 2..17 form four epilogue groups that take every fourth tile: each
//     thread reads one accumulator row with tcgen05.ld and quantizes it
//     group by group in registers (min/max, fp16 scale and zero, codes
//     packed four per byte) and writes the row into the packed cache (or
//     the fp16 sink rows, or fp32 rows for the test export).
//
// One persistent CTA per SM walks a contiguous range of tiles.  Jobs are
// ordered (head, K|V) first and sequence last, so consecutive jobs share
// their rotation.  R's fp16 halves live in shared memory in the MMA's
// K-major swizzled layout; when the range moves to a job with another
// rotation, the epilogue group that finished the previous job's last tile
// rewrites them (every MMA before it has completed by then) and releases
// the MMA warp.  The FWHT operand needs half the room, so there two are
// resident: the first two rotations of the range are written at the start
// by two groups at once, and the group that finishes rotation n's last tile
// writes rotation n + 2 into the buffer n used, a whole rotation ahead of
// its first MMA.  Every wait is bounded: a wait that gives up sets
// KVQ_DEV_TIMEOUT and the CTA stops.
//
// Permutation + FWHT rotation ("RotateKV", abstract item (i); "KVLinC",
// abstract: Hadamard rotation) is the same contraction with
// R = P . H / sqrt(128): y = x[perm] transformed by the Sylvester Hadamard
// matrix H is x . B with B[m][j] = H[pinv[m]][j] = (-1)^popcount(pinv[m] & j),
// pinv the inverse permutation.  B's entries are +-1, exact in fp16, so one
// MMA pass (no lo part) gives the transform exactly up to fp32 accumulation,
// and the epilogue multiplies by 1/sqrt(128) in fp32 like the CUDA-core
// FWHT does.  B is built in shared memory from the permutation (no R in
// memory).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "kvq_internal.cuh"

namespace kvq {
namespace tc {

constexpr int TILE_M = 128;                    // rows (tokens) per tile = MMA M
constexpr int A_STAGES = 3;
constexpr int A_HALF = TILE_M * 128;           // one 64-column half of an x tile (16 KB)
constexpr int A_BYTES = 2 * A_HALF;            // 32 KB
constexpr int B_HALF = D * 128;                // one 64-column (K) half of R^T (16 KB)
constexpr int B_PART = 2 * B_HALF;             // R_hi or R_lo (32 KB)
constexpr int EPI_GROUPS = 4;                  // epilogue groups = accumulators in flight
constexpr int EPI_WARPS = 4 * EPI_GROUPS;
constexpr int THREADS = 32 * (2 + EPI_WARPS);  // 576
constexpr uint32_t TMEM_COLS = 128 * EPI_GROUPS;   // one 128-column fp32 accumulator per group

// shared memory (offsets from a 1024-byte aligned base)
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + A_STAGES * A_BYTES;
constexpr int OFF_PINV = OFF_B + 2 * B_PART;  // FWHT: per epilogue warp, 128 B of scratch
// barriers: full_a[A_STAGES], empty_a[A_STAGES], acc_full[EPI_GROUPS],
// acc_empty[EPI_GROUPS], b_ready[2] (one per B buffer)
constexpr int BAR_FULL = 0, BAR_EMPTY = A_STAGES, BAR_ACCF = 2 * A_STAGES,
              BAR_ACCE = 2 * A_STAGES + EPI_GROUPS, BAR_BREADY = 2 * A_STAGES + 2 * EPI_GROUPS,
              NBAR = 2 * A_STAGES + 2 * EPI_GROUPS + 2;
constexpr int OFF_BAR = OFF_PINV + 128 * EPI_WARPS;
constexpr int OFF_TMEMPTR = OFF_BAR + 8 * NBAR;
constexpr int OFF_ABORT = OFF_TMEMPTR + 16;
constexpr int SMEM_USED = OFF_ABORT + 16;
constexpr int SMEM_BYTES = SMEM_USED + 1024;   // slack for aligning the base

// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), A and
// B fp16 (bits 7-9, 10-12 = 0), both K-major (bits 15, 16 = 0), N >> 3 at
// bit 17, M >> 4 at bit 24.
constexpr uint32_t IDESC = (1u << 4) | ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(TILE_M >> 4) << 24);

// Shared-memory matrix descriptor, K-major with 128-byte swizzle: start
// address >> 4 (bits 0-13), leading byte offset 1 (unused by this layout,
// bits 16-29), stride byte offset 1024 >> 4 between 8-row groups (bits
// 32-45), descriptor version 1 (bits 46-47), layout 2 = 128-byte swizzle
// (bits 61-63).  Rows are 128 bytes; a K step of 16 fp16 advances the start
// address by 32 bytes inside the 1024-byte swizzle atom.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate), "r"(0u), "r"(0u),
        "r"(0u), "r"(0u)
        : "memory");
}

// Arrive (once) on `bar` when every tcgen05 operation this thread issued
// before has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

// 3-D tiled TMA load of box {64, 1, 128} at coordinates (c0, c1, c2) into
// this CTA's own 1024-byte aligned shared memory, completion on `bar`.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

}  // namespace tc

// Work of one launch.  Cache mode: job j = (2h + kind)*B + b over
// x = K (kind 0) or V (kind 1) of sequence b, rows t in [0, T); its
// rotation key is j / B = 2h + kind.  Test mode (out_f32 set): one job,
// x = [N][128], R = R0 (or perm = one plane of 128), fp32 rows out.
struct TcArgs {
    const float *R0, *R1;   // dense: R_k, R_v [Hkv][128][128]
    const int32_t *perm;    // FWHT: [2][Hkv][128] (cache) or [128] (test); else nullptr
    float *out_f32;         // test mode output [T][128], else nullptr
    int T;                  // rows per job
    int B;                  // sequences (1 in test mode)
    int Hkv;
    int tiles_per_job, ntiles, tiles_per_cta;
};

// R^T of one job in the B operand layout: row j (output column), K index i
// (input element); fp16 hi and lo parts.  128 threads, thread tt = row j;
// each writes 16-byte chunks (8 consecutive i), conflict-free under the
// swizzle (chunk c of row j sits at chunk position c ^ (j & 7)).
__device__ __forceinline__ void convert_r(const float *R, uint8_t *bhi, uint8_t *blo, int tt) {
    const int j = tt;
#pragma unroll 4
    for (int cc = 0; cc < 16; cc++) {
        const int i0 = 8 * cc;
        float r[8];
#pragma unroll
        for (int e = 0; e < 8; e++) r[e] = R[(size_t)(i0 + e) * D + j];
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const __half h0 = __float2half_rn(r[2 * e]), h1 = __float2half_rn(r[2 * e + 1]);
            const __half l0 = __float2half_rn(__fsub_rn(r[2 * e], __half2float(h0)));
            const __half l1 = __float2half_rn(__fsub_rn(r[2 * e + 1], __half2float(h1)));
            hw[e] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
            lw[e] = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
        }
        const int kb = i0 >> 6, ch = (i0 & 63) >> 3;
        const int off = kb * tc::B_HALF + j * 128 + ((ch ^ (j & 7)) << 4);
        *reinterpret_cast<uint4 *>(bhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4 *>(blo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
}

// P . H of one job in the same B layout (row j, K index m), entries
// (-1)^popcount(pinv[m] & j) as fp16 +-1, pinv the inverse permutation.
// Called by the 128 threads of one epilogue group, thread tt = row j.  Each
// warp inverts the permutation into its own 128 bytes of scratch (pinv_w),
// so only warp-level synchronisation is needed.  Entries of a permutation
// outside [0, 128) are wrapped.
__device__ __forceinline__ void build_fwht_b(const int4 pv, uint8_t *bhi, uint8_t *pinv_w,
                                             int tt) {
    const int lane = tt & 31;
    // pv = perm[lane], perm[lane + 32], perm[lane + 64], perm[lane + 96]
    pinv_w[pv.x & (D - 1)] = (uint8_t)lane;
    pinv_w[pv.y & (D - 1)] = (uint8_t)(lane + 32);
    pinv_w[pv.z & (D - 1)] = (uint8_t)(lane + 64);
    pinv_w[pv.w & (D - 1)] = (uint8_t)(lane + 96);
    __syncwarp();
    const int j = tt;
#pragma unroll 4
    for (int cc = 0; cc < 16; cc++) {
        const int m0 = 8 * cc;
        const uint2 pw = *reinterpret_cast<const uint2 *>(pinv_w + m0);   // pinv[m0 .. m0+7]
        uint32_t hw[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const uint32_t w = e < 2 ? pw.x : pw.y;
            const uint32_t p0 = (w >> (16 * (e & 1))) & 0xffu, p1 = (w >> (16 * (e & 1) + 8)) & 0xffu;
            const uint32_t s0 = __popc(p0 & (uint32_t)j) & 1u, s1 = __popc(p1 & (uint32_t)j) & 1u;
            hw[e] = (0x3C00u | (s0 << 15)) | ((0x3C00u | (s1 << 15)) << 16);
        }
        const int kb = m0 >> 6, ch = (m0 & 63) >> 3;
        const int off = kb * tc::B_HALF + j * 128 + ((ch ^ (j & 7)) << 4);
        *reinterpret_cast<uint4 *>(bhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
    // every lane has read pinv_w before a later build rewrites it
    __syncwarp();
}

// The permutation entries of rotation key hk (cache: 2h + kind; test: 0)
// that lane `lane` of a building warp needs (FWHT mode); loaded ahead of the
// wait that precedes the build.
__device__ __forceinline__ int4 fwht_perm_regs(const TcArgs &a, bool to_cache, int hk, int lane) {
    const int32_t *pm = to_cache ? a.perm + ((size_t)(hk & 1) * a.Hkv + (hk >> 1)) * D : a.perm;
    return make_int4(pm[lane], pm[lane + 32], pm[lane + 64], pm[lane + 96]);
}

// The B operand of rotation key hk (cache: 2h + kind; test: 0), written by
// the 128 threads of one epilogue group (gt = thread in the group) into the
// buffer at dst: dense, R_hi at dst and R_lo at dst + B_PART; FWHT, the +-1
// matrix at dst.  pv: fwht_perm_regs of hk; pinv_w: the warp's 128 bytes of
// scratch (FWHT mode).
__device__ __forceinline__ void load_b(const TcArgs &a, bool to_cache, int hk, int4 pv,
                                       uint8_t *dst, uint8_t *pinv_w, int gt) {
    if (a.perm) {
        build_fwht_b(pv, dst, pinv_w, gt);
    } else {
        const float *R = to_cache ? ((hk & 1) ? a.R1 : a.R0) + (size_t)(hk >> 1) * D * D : a.R0;
        convert_r(R, dst, dst + tc::B_PART, gt);
    }
}

// The epilogue quantizes one row per thread with quantize_group_thread
// (kvq_internal.cuh), group by group.

template <bool TO_CACHE, bool FWHT>
__global__ void __launch_bounds__(tc::THREADS, 1)
    append_dense_tc_kernel(const __grid_constant__ CUtensorMap mapK,
                           const __grid_constant__ CUtensorMap mapV, TcArgs a, CacheDst c) {
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);   // 1024-B aligned base
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + OFF_TMEMPTR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_ABORT);
    // B buffers: the dense operand (hi + lo) fills both halves of the B
    // region; the FWHT operand (hi only) takes one half, so two rotations
    // can be resident and the next one is built ahead of its first tile.
    constexpr int NBUF = FWHT ? 2 : 1;
    auto bbuf = [&](int x) { return smem + OFF_B + x * B_PART; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int k0 = blockIdx.x * a.tiles_per_cta;
    const int nmy = max(0, min(a.ntiles, k0 + a.tiles_per_cta) - k0);
    auto job_of = [&](int k) { return k / a.tiles_per_job; };
    auto rot_of = [&](int k) { return job_of(k) / a.B; };     // rotation key 2h + kind
    // tile k takes another rotation than tile k - 1 (divisions only at job
    // boundaries)
    auto new_rot = [&](int k) { return job_of(k) != job_of(k - 1) && rot_of(k) != rot_of(k - 1); };
    // this CTA's rotations are rk0 .. rk_last, consecutive keys; the n-th
    // (key rk0 + n) lives in B buffer n % NBUF, whose b_ready barrier
    // completes its phase n / NBUF when the operand is written
    const int rk0 = nmy > 0 ? rot_of(k0) : 0, rk_last = nmy > 0 ? rot_of(k0 + nmy - 1) : -1;
    auto fail = [&]() {
        set_status(c.status, KVQ_DEV_TIMEOUT);
        *abort_flag = 1;
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < A_STAGES; i++) {
            mbar_init(&bar[BAR_FULL + i], 1);
            mbar_init(&bar[BAR_EMPTY + i], 1);
        }
        for (int i = 0; i < EPI_GROUPS; i++) {
            mbar_init(&bar[BAR_ACCF + i], 1);
            mbar_init(&bar[BAR_ACCE + i], 4);       // the four warps of an epilogue group
        }
        for (int i = 0; i < 2; i++) mbar_init(&bar[BAR_BREADY + i], 4);   // one group's 4 warps
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {   // TMEM for the two accumulators (whole warp, .sync.aligned)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_ptr)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ---- producer: x tiles by TMA
        if (lane == 0) {
            int i = 0;
            for (; i < nmy && !*abort_flag; i++) {
                const int k = k0 + i, s = i % A_STAGES, j = job_of(k);
                if (i >= A_STAGES &&
                    !mbar_wait_bounded(&bar[BAR_EMPTY + s], ((i / A_STAGES) - 1) & 1)) {
                    fail();
                    break;
                }
                int kind = 0, h = 0, row = (k - j * a.tiles_per_job) * TILE_M;
                if (TO_CACHE) {
                    const int hk = j / a.B;
                    kind = hk & 1;
                    h = hk >> 1;
                    row += (j - hk * a.B) * a.T;       // + b * T
                }
                const CUtensorMap *map = kind == 0 ? &mapK : &mapV;
                uint8_t *dst = smem + OFF_A + s * A_BYTES;
                mbar_arrive_expect_tx(&bar[BAR_FULL + s], A_BYTES);
                tma_load_3d(dst, map, 0, h, row, &bar[BAR_FULL + s]);
                tma_load_3d(dst + A_HALF, map, 64, h, row, &bar[BAR_FULL + s]);
            }
            // no copy may still be landing when the CTA exits (after an abort
            // the last stages may not have been consumed): bounded waits
            drain_ring(&bar[BAR_FULL], A_STAGES, max(0, i - A_STAGES), i);
        }
    } else if (warp == 1) {
        // ---- MMA issuer
        if (lane == 0) {
            int nr = -1;   // rotation index (rot - rk0) of the current tile
            int i = 0;
            for (; i < nmy && !*abort_flag; i++) {
                const int k = k0 + i, s = i % A_STAGES, buf = i % EPI_GROUPS;
                if (i == 0 || new_rot(k)) {
                    ++nr;
                    if (!mbar_wait_bounded(&bar[BAR_BREADY + nr % NBUF], (nr / NBUF) & 1)) {
                        fail();
                        break;
                    }
                }
                if (i >= EPI_GROUPS &&
                    !mbar_wait_bounded(&bar[BAR_ACCE + buf], ((i / EPI_GROUPS) - 1) & 1)) {
                    fail();
                    break;
                }
                if (!mbar_wait_bounded(&bar[BAR_FULL + s], (i / A_STAGES) & 1)) { fail(); break; }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * 128);
                const uint32_t abase = smem_u32(smem + OFF_A + s * A_BYTES);
                uint32_t acc = 0;
#pragma unroll
                for (int part = 0; part < (FWHT ? 1 : 2); part++) {
                    const uint32_t bbase = smem_u32(bbuf(nr % NBUF) + part * B_PART);
#pragma unroll
                    for (int kb = 0; kb < 2; kb++)
#pragma unroll
                        for (int ks = 0; ks < 4; ks++) {
                            mma_f16(d, sw128_desc(abase + kb * A_HALF + 32 * ks),
                                    sw128_desc(bbase + kb * B_HALF + 32 * ks), acc);
                            acc = 1;
                        }
                }
                mma_commit(&bar[BAR_EMPTY + s]);      // x stage free once these MMAs are done
                mma_commit(&bar[BAR_ACCF + buf]);     // accumulator ready
            }
            // the accumulators are freed below: the last MMAs must have completed
            if (i > 0)
                mbar_wait_bounded(&bar[BAR_ACCF + (i - 1) % EPI_GROUPS], ((i - 1) / EPI_GROUPS) & 1);
        }
    } else {
        // ---- epilogue groups
        const int eg = (warp - 2) >> 2;                 // group g: warps 2+4g .. 5+4g
        const int gt = threadIdx.x - 64 - 128 * eg;     // 0..127 within the group
        const int q = warp & 3;                         // TMEM lane quarter this warp may read
        const int row = 32 * q + lane;                  // accumulator row = tile row
        uint8_t *pinv_w = smem + OFF_PINV + 128 * (warp - 2);
        // the first NBUF rotations: group n writes rotation n
        if (eg < NBUF && rk0 + eg <= rk_last) {
            const int hk = rk0 + eg;
            load_b(a, TO_CACHE, hk, FWHT ? fwht_perm_regs(a, TO_CACHE, hk, lane) : make_int4(0, 0, 0, 0),
                   bbuf(eg), pinv_w, gt);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[BAR_BREADY + eg]);
        }
        int cur_job = -1, L0 = -1;
        int s_n = 0, s_last = -1;                       // identified sinks of the job's sequence
        for (int i = eg; i < nmy; i += EPI_GROUPS) {
            // decisions stay warp-uniform: tcgen05.ld below is .sync.aligned
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const int k = k0 + i, j = job_of(k), buf = i % EPI_GROUPS;     // = eg
            // global reads this tile needs, issued before the wait on its
            // accumulator: the permutation entries of the rotation it
            // writes next (when it is its rotation's last tile and one more
            // rotation follows beyond the resident ones) and the job's
            // start length
            const bool rebuild = i + 1 < nmy && new_rot(k + 1) && rot_of(k) + NBUF <= rk_last;
            const int hk_next = rot_of(k) + NBUF;
            int4 pv = make_int4(0, 0, 0, 0);
            if (FWHT && rebuild) pv = fwht_perm_regs(a, TO_CACHE, hk_next, lane);
            int b = 0, h = 0, kind = 0;
            if (TO_CACHE) {
                const int hk = j / a.B;
                kind = hk & 1;
                h = hk >> 1;
                b = j - hk * a.B;
                if (j != cur_job) {
                    L0 = start_len_thread(c, b, kind == 0 && h == 0 && gt == 0);
                    sink_list_end(c, b, s_n, s_last);
                    cur_job = j;
                }
            }
            if (!__all_sync(0xffffffffu,
                            mbar_wait_bounded(&bar[BAR_ACCF + buf], (i / EPI_GROUPS) & 1))) {
                fail();
                break;
            }
            tc_fence_after();
            // this tile's MMAs (and all earlier ones) are done, so no MMA reads
            // its rotation's buffer any more: the rotation NBUF further on
            // goes into it now
            if (rebuild) {
                const int x = (rot_of(k) - rk0) % NBUF;
                load_b(a, TO_CACHE, hk_next, pv, bbuf(x), pinv_w, gt);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[BAR_BREADY + x]);
            }
            const int t = (k - j * a.tiles_per_job) * TILE_M + row;
            const bool valid = t < a.T && (!TO_CACHE || L0 >= 0);
            const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * 128);
            const int p = L0 + t;
            const int srow = TO_CACHE && valid ? sink_row_after(c, b, p, s_n, s_last) : -1;
            const bool sink = srow >= 0;
            uint32_t words[8] = {0, 0, 0, 0, 0, 0, 0, 0}, meta[4] = {0, 0, 0, 0};
#pragma unroll 1
            for (int g = 0; g < NG; g++) {
                float v[32];
                tmem_ld32(taddr + 32 * g, v);
                if (FWHT) scale_group(v, 0.08838834764831845f);   // the FWHT's 1/sqrt(128), in fp32
                if (g == NG - 1) {
                    // the accumulator is no longer needed: free it for the tile after next
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar[BAR_ACCE + buf]);
                }
                if (!valid) continue;
                if (!TO_CACHE) {
                    float *dst = a.out_f32 + (size_t)t * D + 32 * g;
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4 *>(dst + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                } else if (sink) {
                    uint16_t *dst = (kind == 0 ? c.k_sink : c.v_sink) +
                                    (((size_t)b * c.Hkv + h) * c.S + (size_t)srow) * D + 32 * g;
#pragma unroll
                    for (int e = 0; e < 32; e += 8)
                        *reinterpret_cast<uint4 *>(dst + e) =
                            make_uint4(pack_half2(v[e], v[e + 1]), pack_half2(v[e + 2], v[e + 3]),
                                       pack_half2(v[e + 4], v[e + 5]), pack_half2(v[e + 6], v[e + 7]));
                } else {
                    meta[g] = quantize_group_thread(v, g, words);
                }
            }
            const long long bix =
                TO_CACHE && valid
                    ? cache_block_index(c.table, c.num_blocks, c.nblk, c.Hkv, b, h, p / BLK_TOK)
                    : 0;
            if (bix < 0) set_status(c.status, KVQ_DEV_BAD_TABLE);
            if (sink && c.sink_pos && kind == 0) {
#pragma unroll
                for (int g = 0; g < NG; g++) meta[g] = SINK_KMETA_MARK;
            }
            if (TO_CACHE && valid && bix >= 0) {
                // sink rows leave zero codes and metadata in their cache slots
                // (an identified sink: the marker in its K meta)
                uint8_t *block = c.blocks + (size_t)bix * BLK_BYTES;
                const int tau = p % BLK_TOK;
                if (kind == 0) {
#pragma unroll
                    for (int w = 0; w < 8; w++)
                        *reinterpret_cast<uint32_t *>(block + off_kword(tau, w)) = words[w];
#pragma unroll
                    for (int g = 0; g < NG; g++)
                        *reinterpret_cast<uint32_t *>(block + off_kmeta(tau, g)) = meta[g];
                } else {
#pragma unroll
                    for (int w = 0; w < 16; w++)
                        *reinterpret_cast<uint16_t *>(block + off_vpiece(tau, w)) =
                            (uint16_t)(words[w >> 1] >> (16 * (w & 1)));
#pragma unroll
                    for (int g = 0; g < NG; g++)
                        *reinterpret_cast<uint32_t *>(block + off_vmeta(tau, g)) = meta[g];
                }
            }
        }
    }

    // ---- teardown: every role is done; warp 1 frees TMEM
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS)
                     : "memory");
    }
    if (TO_CACHE) append_done(c);
}

// ---- host side ---------------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// x viewed as [rows][Hkv][128] fp16: dims {128, Hkv, rows}, box {64, 1, 128},
// 128-byte swizzle; rows past the end read as zeros.
bool make_map(CUtensorMap *m, const uint16_t *X, int Hkv, long long rows) {
    const auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)tc::TILE_M};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<uint16_t *>(X), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool TO_CACHE, bool FWHT>
cudaError_t launch_tc(const CUtensorMap &mk, const CUtensorMap &mv, TcArgs a, const CacheDst &c,
                      cudaStream_t st) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int grid = std::max(1, std::min(sms, a.ntiles));
    a.tiles_per_cta = (a.ntiles + grid - 1) / grid;
    e = cudaFuncSetAttribute(append_dense_tc_kernel<TO_CACHE, FWHT>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(append_dense_tc_kernel<TO_CACHE, FWHT>, dim3(grid), dim3(tc::THREADS),
                      (size_t)tc::SMEM_BYTES, st, mk, mv, a, c);
}

}  // namespace

// Which appends take this kernel rather than the CUDA-core ones, from their
// crossovers measured on B200 (32 KV heads, L2 flushed before each call):
// a dense rotation from 32 new tokens per sequence, or from 8 when the batch
// brings at least 256 rows (below that the CUDA-core kernel, which shares one
// fetch of R among several sequences, wins); the permutation + FWHT form,
// whose CUDA-core kernels do far less arithmetic, from 128 tokens, or from
// 32 when the batch brings at least 1024 rows.  A job shorter than a tile
// loads 128 rows and drops those past its own T.
bool append_tc_eligible(int mode, const uint16_t *K, const uint16_t *V, int T, int B) {
    const auto al = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    const long long rows = (long long)B * T;
    const bool worth = mode == KVQ_ROT_DENSE ? (T >= 32 || (T >= 8 && rows >= 256))
                                             : (T >= 128 || (T >= 32 && rows >= 1024));
    return worth && al(K) && al(V) && encode_fn() != nullptr;
}

cudaError_t launch_append_tc(const uint16_t *K, const uint16_t *V, int T, int mode,
                             const float *R_k, const float *R_v, const int32_t *perm,
                             const kvq_cache_desc &cd, int32_t *seq_lens, cudaStream_t st) {
    CUtensorMap mk, mv;
    const long long rows = (long long)cd.B * T;
    if (!make_map(&mk, K, cd.Hkv, rows) || !make_map(&mv, V, cd.Hkv, rows)) return cudaErrorInvalidValue;
    const CacheDst c = cache_dst(cd, seq_lens, T);
    TcArgs a;
    a.R0 = R_k;
    a.R1 = R_v;
    a.perm = mode == KVQ_ROT_DENSE ? nullptr : perm;
    a.out_f32 = nullptr;
    a.T = T;
    a.B = cd.B;
    a.Hkv = cd.Hkv;
    a.tiles_per_job = (T + tc::TILE_M - 1) / tc::TILE_M;
    a.ntiles = a.tiles_per_job * cd.B * cd.Hkv * 2;
    a.tiles_per_cta = 0;
    return a.perm ? launch_tc<true, true>(mk, mv, a, c, st) : launch_tc<true, false>(mk, mv, a, c, st);
}

cudaError_t launch_debug_rotate_tc(const uint16_t *X, int N, int mode, const float *R,
                                   const int32_t *perm, float *out, cudaStream_t st) {
    CUtensorMap m;
    if (!make_map(&m, X, 1, N)) return cudaErrorInvalidValue;
    CacheDst c{};
    TcArgs a;
    a.R0 = a.R1 = R;
    a.perm = mode == KVQ_ROT_DENSE ? nullptr : perm;
    a.out_f32 = out;
    a.T = N;
    a.B = 1;
    a.Hkv = 1;
    a.tiles_per_job = (N + tc::TILE_M - 1) / tc::TILE_M;
    a.ntiles = a.tiles_per_job;
    a.tiles_per_cta = 0;
    return a.perm ? launch_tc<false, true>(m, m, a, c, st) : launch_tc<false, false>(m, m, a, c, st);
}

}  // namespace kvq
