// Decode attention over the packed INT2 cache.
//
// Method: the query is rotated by the key rotation (so q.k is unchanged up
// to quantization), the attention is the standard scaled-dot-product softmax
// over the dequantised cache, and the value rotation is removed after the
// attention ("Output-Aware Rotation for INT2 KV-Cache Quantization", section
// "Key Details"; "Why It Matters": the attention itself is unchanged).
// Sinks are the leading positions stored in fp16 ("RotateKV", abstract item
// (iii)).
//
// Three kernels:
//   decode_prologue_kernel  per (b, query head): q_rot = q.R_k (or perm+FWHT),
//                           scaled into the exp2 domain; sink-token partial
//                           softmax in fp32; block 0 also writes the prefix
//                           sums that balance the split kernel.
//   decode_split_kernel<G>  stream-K over all cache blocks of all (b, h)
//                           units: every CTA takes an equal share of 16-token
//                           blocks.  A producer warp streams them into a
//                           shared-memory ring with 1-D bulk copies (TMA);
//                           four consumer warps run the scores and P.V on
//                           tensor cores straight from the packed codes and
//                           keep an online softmax; each (CTA, unit) segment
//                           leaves one partial (m, l, o_rot[128]) per head.
//   decode_merge_kernel     per (b, query head): merge the partials, then
//                           out = o_rot . R_v^T (or FWHT + inverse permutation).
//
// Tensor-core operand trick.  A 2-bit code c sitting in bits [2g, 2g+1] of a
// 16-bit lane, with every other bit zero, IS the fp16 subnormal c*4^g*2^-24.
// So one AND turns a packed word into an m16n8k16 fragment register (two
// codes); the 4^g*2^-24 factor is folded into a per-group fp32 scale
// afterwards.  Products and sums stay exact or fp32: the query enters as an
// fp16 hi/lo pair (two N columns), the softmax weights times V scales as fp16.
// The dequantisation c*s + z is factored: sum_j q_j (c_j s + z) =
// s*sum_j q_j c_j + z*sum_j q_j, so only the integer codes go through the MMA.
#include "kvq_internal.cuh"

namespace kvq {

constexpr int DEC_CONSUMER_WARPS = 4;
constexpr int DEC_THREADS = 32 * (DEC_CONSUMER_WARPS + 1);
constexpr int STAGE_BLKS = 2 * DEC_CONSUMER_WARPS;        // 8 blocks = 128 tokens
constexpr int STAGE_BYTES = STAGE_BLKS * BLK_BYTES;       // 12 KB
constexpr int NSTAGE = 4;
constexpr int QP = 132;     // per (b, hq): q_s[128] then sum of q_s per group [4]
constexpr int PART = 132;   // per partial: m, l, 0, 0, o[128]
constexpr float LOG2E = 1.4426950408889634f;
#define NEG_INF (__int_as_float(0xff800000))

struct DecodeArgs {
    const uint16_t *Q;
    const uint8_t *blocks;
    const uint16_t *k_sink, *v_sink;
    const float *R_k, *R_v;
    const int32_t *perm;
    const int32_t *seq_lens;
    int32_t *status;
    int32_t *prefix;   // [B+1] workspace
    float *qprep;      // [B*Hq][QP]
    float *sinkp;      // [B*Hq][PART]
    float *part;       // [(C+U)*G][PART]
    uint16_t *out;
    int B, Hq, Hkv, G, S, capacity, nblk, mode, C;
};

// Blocks of 16 tokens that hold codes for a sequence of length L: positions
// [S, L) live in cache blocks S/16 .. (L-1)/16.
__device__ __forceinline__ int unit_blocks(int L, int S, int capacity) {
    if (L < 1 || L > capacity || L <= S) return 0;
    return (L - 1) / BLK_TOK - S / BLK_TOK + 1;
}

// ---------------------------------------------------------------------------------------------
// Prologue.
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128) decode_prologue_kernel(DecodeArgs a) {
    __shared__ __align__(16) float qs[D];
    __shared__ float ssc[MAX_SINK];
    const int hq = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int h = hq / a.G;
    const uint16_t *q = a.Q + ((size_t)b * a.Hq + hq) * D;

    if (blockIdx.x == 0 && blockIdx.y == 0) {
        // prefix[b+1] = prefix[b] + Hkv * blocks(b): chunked scan, 128 threads
        __shared__ int part[128];
        const int per = (a.B + 127) / 128;
        int s = 0;
        for (int i = t * per; i < min(a.B, (t + 1) * per); i++)
            s += a.Hkv * unit_blocks(a.seq_lens[i], a.S, a.capacity);
        part[t] = s;
        __syncthreads();
        if (t == 0) {
            int acc = 0;
            for (int i = 0; i < 128; i++) {
                const int v = part[i];
                part[i] = acc;
                acc += v;
            }
        }
        __syncthreads();
        int acc = part[t];
        for (int i = t * per; i < min(a.B, (t + 1) * per); i++) {
            a.prefix[i] = acc;
            const int L = a.seq_lens[i];
            if (L < 1 || L > a.capacity) set_status(a.status, KVQ_DEV_BAD_LEN);
            acc += a.Hkv * unit_blocks(L, a.S, a.capacity);
        }
        if (t == 127) a.prefix[a.B] = acc;
        __syncthreads();
    }

    // q_rot in fp32, then scaled by log2(e)/sqrt(128) so scores are exp2 exponents
    float qr;
    if (a.mode == KVQ_ROT_DENSE) {
        __shared__ float qin[D];
        qin[t] = __half2float(__ushort_as_half(q[t]));
        __syncthreads();
        const float *R = a.R_k + (size_t)h * D * D;
        float acc = 0.f;
#pragma unroll 8
        for (int i = 0; i < D; i++) acc = fmaf(qin[i], R[i * D + t], acc);
        qr = acc;
        qs[t] = qr;
    } else {
        if (warp == 0) {
            __shared__ uint16_t xq[D];
            *reinterpret_cast<uint2 *>(&xq[4 * lane]) = *reinterpret_cast<const uint2 *>(q + 4 * lane);
            const int4 pi = *reinterpret_cast<const int4 *>(a.perm + (size_t)h * D + 4 * lane);
            __syncwarp();
            float v[4] = {__half2float(__ushort_as_half(xq[pi.x & (D - 1)])),
                          __half2float(__ushort_as_half(xq[pi.y & (D - 1)])),
                          __half2float(__ushort_as_half(xq[pi.z & (D - 1)])),
                          __half2float(__ushort_as_half(xq[pi.w & (D - 1)]))};
            fwht128_warp(v);
            *reinterpret_cast<float4 *>(&qs[4 * lane]) =
                make_float4(v[0] * 0.08838834764831845f, v[1] * 0.08838834764831845f,
                            v[2] * 0.08838834764831845f, v[3] * 0.08838834764831845f);
        }
    }
    __syncthreads();
    const float qscale = LOG2E * 0.08838834764831845f;
    const float qv = qs[t] * qscale;
    float *qp = a.qprep + ((size_t)b * a.Hq + hq) * QP;
    qp[t] = qv;
    float gs = qv;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) gs += __shfl_xor_sync(0xffffffffu, gs, off);
    if (lane == 0) qp[D + warp] = gs;

    // sink partial (fp32, CUDA cores): at most MAX_SINK tokens
    if (a.S > 0) {
        __syncthreads();
        qs[t] = qv;
        __syncthreads();
        const int L = a.seq_lens[b];
        const bool ok = (L >= 1 && L <= a.capacity);
        const int ns = ok ? min(a.S, L) : 0;
        const uint16_t *ks = a.k_sink + ((size_t)b * a.Hkv + h) * a.S * D;
        const uint16_t *vs = a.v_sink + ((size_t)b * a.Hkv + h) * a.S * D;
        for (int tk = warp; tk < ns; tk += 4) {
            const uint2 u = *reinterpret_cast<const uint2 *>(ks + (size_t)tk * D + 4 * lane);
            const float2 k01 = unpack_half2(u.x), k23 = unpack_half2(u.y);
            float d = qs[4 * lane] * k01.x + qs[4 * lane + 1] * k01.y + qs[4 * lane + 2] * k23.x +
                      qs[4 * lane + 3] * k23.y;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
            if (lane == 0) ssc[tk] = d;
        }
        __syncthreads();
        float m = NEG_INF;
        for (int tk = 0; tk < ns; tk++) m = fmaxf(m, ssc[tk]);
        float l = 0.f, o = 0.f;
        for (int tk = 0; tk < ns; tk++) {
            const float p = exp2f(ssc[tk] - m);
            l += p;
            o = fmaf(p, __half2float(__ushort_as_half(vs[(size_t)tk * D + t])), o);
        }
        float *sp = a.sinkp + ((size_t)b * a.Hq + hq) * PART;
        sp[4 + t] = o;
        if (t == 0) {
            sp[0] = m;
            sp[1] = l;
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Split kernel.
// ---------------------------------------------------------------------------------------------
// Per-CTA schedule over the global block space: unit u = b*Hkv + h holds
// nb(b) consecutive global blocks starting at prefix[b] + h*nb(b).
struct Sched {
    int b, h, nb, ustart, cur, end;
};

__device__ __forceinline__ void sched_fix_unit(Sched &s, const DecodeArgs &a) {
    // move (b, h) forward until cur lies inside the unit
    while (s.cur >= s.ustart + s.nb && s.cur < s.end) {
        if (++s.h == a.Hkv) {
            s.h = 0;
            ++s.b;
        }
        if (s.h == 0) s.nb = (a.prefix[s.b + 1] - a.prefix[s.b]) / a.Hkv;
        s.ustart = a.prefix[s.b] + s.h * s.nb;
    }
}

__device__ __forceinline__ bool sched_init(Sched &s, const DecodeArgs &a) {
    const int N = a.prefix[a.B];
    const int W = max(1, (N + a.C - 1) / a.C);
    s.cur = blockIdx.x * W;
    s.end = min(N, s.cur + W);
    if (s.cur >= s.end) return false;
    int lo = 0, hi = a.B;            // largest b with prefix[b] <= cur
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (a.prefix[mid] <= s.cur) lo = mid; else hi = mid;
    }
    s.b = lo;
    s.nb = (a.prefix[s.b + 1] - a.prefix[s.b]) / a.Hkv;
    while (s.nb == 0) {              // empty sequences have prefix[b] == prefix[b+1]
        ++s.b;
        s.nb = (a.prefix[s.b + 1] - a.prefix[s.b]) / a.Hkv;
    }
    s.h = (s.cur - a.prefix[s.b]) / s.nb;
    s.ustart = a.prefix[s.b] + s.h * s.nb;
    return true;
}

template <int G>
struct Cfg {
    static constexpr int NTK = G;                    // K-side N tiles (8G columns)
    static constexpr int NTK_STEP = G >= 8 ? 2 : 1;  // N tiles one K step touches
    static constexpr int NTV = G <= 2 ? 1 : G / 2;   // V-side N tiles (4G columns)
    static constexpr int HPL = G >= 8 ? 2 : 1;       // heads whose scores a lane holds
};

// group of K-side N tile nu for lane quad-index c
template <int G>
__device__ __forceinline__ int ktile_group(int nu, int c) {
    return ((8 * nu + 2 * c) / (2 * G));
}
template <int G>
__device__ __forceinline__ int ktile_head(int nu, int c) {
    return ((8 * nu + 2 * c) % (2 * G)) / 2;
}
template <int G>
__device__ __forceinline__ int lane_head(int c, int hh) {
    return G == 1 ? 0 : (G == 2 ? (c & 1) : (G == 4 ? c : 4 * hh + c));
}
// arr[idx] for a runtime idx without dynamic register indexing
template <int N>
__device__ __forceinline__ float pick(const float (&arr)[N], int idx) {
    float v = arr[0];
#pragma unroll
    for (int i = 1; i < N; i++)
        if (idx == i) v = arr[i];
    return v;
}
// head slot of K-side N tile nu
template <int G>
__device__ __forceinline__ int ktile_slot(int nu) {
    return G >= 8 ? (nu & 1) : 0;
}
// element index inside a group fed by MMA k-slot kappa of a K step with byte
// offset delta (0: bytes 4w, 4w+2 ; 1: bytes 4w+1, 4w+3 of a 32-bit word)
__device__ __forceinline__ int kslot_elem(int kappa, int delta) {
    return 4 * ((kappa >> 1) & 3) + 16 * (kappa >> 3) + 2 * (kappa & 1) + delta;
}

template <int G>
__global__ void __launch_bounds__(DEC_THREADS, 3) decode_split_kernel(DecodeArgs a) {
    using C = Cfg<G>;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *ring = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + NSTAGE * STAGE_BYTES);
    uint64_t *empty = full + NSTAGE;
    float *fo = reinterpret_cast<float *>(empty + NSTAGE);          // [4][G][128]
    float *fm = fo + DEC_CONSUMER_WARPS * G * D;                     // [4][G]
    float *fl = fm + DEC_CONSUMER_WARPS * G;                         // [4][G]
    float *fz = fl + DEC_CONSUMER_WARPS * G;                         // [4][G][4]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(fz + DEC_CONSUMER_WARPS * G * 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], DEC_CONSUMER_WARPS);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    Sched sc;
    if (!sched_init(sc, a)) return;

    // ------------------------------------------------------------------ producer
    if (warp == DEC_CONSUMER_WARPS) {
        if (lane == 0) {
            int it = 0;
            const int fb = a.S / BLK_TOK;
            while (sc.cur < sc.end) {
                sched_fix_unit(sc, a);
                const int n = min(min(STAGE_BLKS, sc.end - sc.cur), sc.ustart + sc.nb - sc.cur);
                const int s = it % NSTAGE;
                if (!mbar_wait_bounded(&empty[s], ((it / NSTAGE) & 1) ^ 1)) {
                    set_status(a.status, KVQ_DEV_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                const size_t unit = (size_t)sc.b * a.Hkv + sc.h;
                const uint8_t *src =
                    a.blocks + (unit * a.nblk + fb + (sc.cur - sc.ustart)) * (size_t)BLK_BYTES;
                mbar_arrive_expect_tx(&full[s], n * BLK_BYTES);
                bulk_g2s(ring + s * STAGE_BYTES, src, n * BLK_BYTES, &full[s]);
                sc.cur += n;
                ++it;
            }
        }
        return;
    }

    // ------------------------------------------------------------------ consumers
    const int r = lane >> 2, c = lane & 3;
    const int fb = a.S / BLK_TOK;
    // per-unit query operands
    uint32_t qB[8][C::NTK_STEP][2];
    float qsum[C::NTK], alpha[C::NTK];
    // online-softmax state
    float m_run[G], l_run[C::HPL], O[8][4], Z[C::NTV];
    int cur_unit = -1;

    auto reset_state = [&]() {
#pragma unroll
        for (int i = 0; i < G; i++) m_run[i] = NEG_INF;
#pragma unroll
        for (int i = 0; i < C::HPL; i++) l_run[i] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; i++)
#pragma unroll
            for (int k = 0; k < 4; k++) O[i][k] = 0.f;
#pragma unroll
        for (int i = 0; i < C::NTV; i++) Z[i] = 0.f;
    };

    auto load_unit = [&](int b, int h) {
        const float *qbase = a.qprep + ((size_t)b * a.Hq + (size_t)h * G) * QP;
        const int n = lane >> 2;
#pragma unroll
        for (int s8 = 0; s8 < 8; s8++) {
            const int g = s8 & 3, delta = s8 >> 2;
#pragma unroll
            for (int j = 0; j < C::NTK_STEP; j++) {
                const int nu = (g * 2 * G) / 8 + j;
                const int col = 8 * nu + n;
                const int gcol = col / (2 * G), head = (col % (2 * G)) / 2, hl = col & 1;
                uint32_t bb[2] = {0u, 0u};
                if (gcol == g) {
                    const float *qh = qbase + (size_t)head * QP + 32 * g;
#pragma unroll
                    for (int part = 0; part < 2; part++) {
                        float vv[2];
#pragma unroll
                        for (int e2 = 0; e2 < 2; e2++) {
                            const float x = qh[kslot_elem(2 * c + 8 * part + e2, delta)];
                            const __half hi = __float2half_rn(x);
                            vv[e2] = hl == 0 ? __half2float(hi)
                                             : __half2float(__float2half_rn(x - __half2float(hi)));
                        }
                        bb[part] = pack_half2(vv[0], vv[1]);
                    }
                }
                qB[s8][j][0] = bb[0];
                qB[s8][j][1] = bb[1];
            }
        }
#pragma unroll
        for (int nu = 0; nu < C::NTK; nu++) {
            const int g = ktile_group<G>(nu, c), head = ktile_head<G>(nu, c);
            qsum[nu] = qbase[(size_t)head * QP + D + g];
            alpha[nu] = __int_as_float((127 + 24 - 2 * g) << 23);   // 2^24 / 4^g
        }
    };

    auto flush = [&](int slot) {
        // reduce l over the 8 row lanes, Z over the 4 column lanes
#pragma unroll
        for (int i = 0; i < C::HPL; i++) {
            l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 4);
            l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 8);
            l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 16);
        }
#pragma unroll
        for (int i = 0; i < C::NTV; i++) {
            Z[i] += __shfl_xor_sync(0xffffffffu, Z[i], 1);
            Z[i] += __shfl_xor_sync(0xffffffffu, Z[i], 2);
        }
        float *wo = fo + warp * G * D;
        if (lane == 0)
#pragma unroll
            for (int i = 0; i < G; i++) fm[warp * G + i] = m_run[i];
        if (lane < 4) {
#pragma unroll
            for (int hh = 0; hh < C::HPL; hh++) {
                const int head = lane_head<G>(lane, hh);
                if (G == 1 ? lane == 0 : (G == 2 ? lane < 2 : true)) fl[warp * G + head] = l_run[hh];
            }
        }
        if (c == 0) {
#pragma unroll
            for (int i = 0; i < C::NTV; i++) {
                const int col = 8 * i + (lane >> 2);
                if (col < 4 * G) fz[(warp * G + col % G) * 4 + col / G] = Z[i];
            }
        }
#pragma unroll
        for (int g = 0; g < 4; g++)
#pragma unroll
            for (int h2 = 0; h2 < 2; h2++)
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const int nv = (g * G) / 8;
                    const int col = 8 * nv + 2 * c + (k & 1);
                    if (col / G == g) {
                        const int head = col % G;
                        const int j = 32 * g + 16 * h2 + 2 * r + (k >> 1);
                        wo[head * D + j] = O[g * 2 + h2][k] * __int_as_float((127 + 24 - 2 * g) << 23);
                    }
                }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * DEC_CONSUMER_WARPS));
        const int tj = threadIdx.x;   // 0..127: element
        for (int head = 0; head < G; head++) {
            float ms = NEG_INF;
#pragma unroll
            for (int w = 0; w < DEC_CONSUMER_WARPS; w++) ms = fmaxf(ms, fm[w * G + head]);
            float acc = 0.f, lsum = 0.f;
#pragma unroll
            for (int w = 0; w < DEC_CONSUMER_WARPS; w++) {
                const float mw = fm[w * G + head];
                const float f = (mw == NEG_INF) ? 0.f : exp2f(mw - ms);
                acc = fmaf(f, fo[(w * G + head) * D + tj] + fz[(w * G + head) * 4 + (tj >> 5)], acc);
                lsum = fmaf(f, fl[w * G + head], lsum);
            }
            float *dst = a.part + ((size_t)slot * G + head) * PART;
            dst[4 + tj] = acc;
            if (tj == 0) {
                dst[0] = ms;
                dst[1] = lsum;
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * DEC_CONSUMER_WARPS));
    };

    reset_state();
    int it = 0;
    while (sc.cur < sc.end) {
        sched_fix_unit(sc, a);
        const int unit = sc.b * a.Hkv + sc.h;
        if (unit != cur_unit) {
            load_unit(sc.b, sc.h);
            cur_unit = unit;
        }
        const int n = min(min(STAGE_BLKS, sc.end - sc.cur), sc.ustart + sc.nb - sc.cur);
        const int L = a.seq_lens[sc.b];
        const int s = it % NSTAGE;
        const bool ok = mbar_wait_bounded(&full[s], (it / NSTAGE) & 1);
        if (!ok || *abort_flag) {
            if (lane == 0) set_status(a.status, KVQ_DEV_TIMEOUT);
            *abort_flag = 1;
            break;
        }
        const int nmine = min(2, max(0, n - 2 * warp));
        float P[2][2][C::HPL];
        float sco[2][2][C::HPL];
        // ---- scores for my (up to) two blocks
#pragma unroll
        for (int bi = 0; bi < 2; bi++) {
#pragma unroll
            for (int st = 0; st < 2; st++)
#pragma unroll
                for (int hh = 0; hh < C::HPL; hh++) sco[bi][st][hh] = NEG_INF;
            if (bi < nmine) {
                const uint8_t *blk = ring + s * STAGE_BYTES + (2 * warp + bi) * BLK_BYTES;
                const uint4 kq = *reinterpret_cast<const uint4 *>(blk + 16 * (4 * r + c));
                float dk[C::NTK][4];
#pragma unroll
                for (int nu = 0; nu < C::NTK; nu++)
#pragma unroll
                    for (int k = 0; k < 4; k++) dk[nu][k] = 0.f;
#pragma unroll
                for (int s8 = 0; s8 < 8; s8++) {
                    const int g = s8 & 3;
                    const uint32_t msk = 0x00030003u << (2 * g);
                    uint32_t a0, a1, a2, a3;
                    if (s8 < 4) {
                        a0 = kq.x & msk; a1 = kq.z & msk; a2 = kq.y & msk; a3 = kq.w & msk;
                    } else {
                        a0 = (kq.x >> 8) & msk; a1 = (kq.z >> 8) & msk;
                        a2 = (kq.y >> 8) & msk; a3 = (kq.w >> 8) & msk;
                    }
#pragma unroll
                    for (int j = 0; j < C::NTK_STEP; j++) {
                        const int nu = (g * 2 * G) / 8 + j;
                        mma16816(dk[nu], a0, a1, a2, a3, qB[s8][j][0], qB[s8][j][1]);
                    }
                }
                // combine groups: s = sum_g sc*(hi+lo)*2^24/4^g + z*sum(q_g)
                float part_sc[2][C::HPL];
#pragma unroll
                for (int st = 0; st < 2; st++)
#pragma unroll
                    for (int hh = 0; hh < C::HPL; hh++) part_sc[st][hh] = 0.f;
#pragma unroll
                for (int nu = 0; nu < C::NTK; nu++) {
                    const int g = ktile_group<G>(nu, c);
                    const uint2 mk = *reinterpret_cast<const uint2 *>(blk + OFF_KM + 8 * (4 * r + g));
                    const float2 sz0 = unpack_half2(mk.x), sz1 = unpack_half2(mk.y);
                    const int hh = ktile_slot<G>(nu);
                    part_sc[0][hh] += sz0.x * ((dk[nu][0] + dk[nu][1]) * alpha[nu]) + sz0.y * qsum[nu];
                    part_sc[1][hh] += sz1.x * ((dk[nu][2] + dk[nu][3]) * alpha[nu]) + sz1.y * qsum[nu];
                }
#pragma unroll
                for (int st = 0; st < 2; st++)
#pragma unroll
                    for (int hh = 0; hh < C::HPL; hh++) {
                        float v = part_sc[st][hh];
                        if (G == 1) {
                            v += __shfl_xor_sync(0xffffffffu, v, 1);
                            v += __shfl_xor_sync(0xffffffffu, v, 2);
                        } else if (G == 2) {
                            v += __shfl_xor_sync(0xffffffffu, v, 2);
                        }
                        const int pos = (fb + (sc.cur - sc.ustart) + 2 * warp + bi) * BLK_TOK + r + 8 * st;
                        sco[bi][st][hh] = (pos >= a.S && pos < L) ? v : NEG_INF;
                    }
            }
        }
        // ---- online softmax update (all lanes of the warp take the same branch)
        if (nmine > 0) {
            float mt[C::HPL];
#pragma unroll
            for (int hh = 0; hh < C::HPL; hh++) {
                float v = fmaxf(fmaxf(sco[0][0][hh], sco[0][1][hh]), fmaxf(sco[1][0][hh], sco[1][1][hh]));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                mt[hh] = v;
            }
            float mnew[G];
            bool grow = false;
#pragma unroll
            for (int hd = 0; hd < G; hd++) {
                // owner lane (quad index) of head hd in the score layout
                const int owner = G == 1 ? 0 : (G == 2 ? (hd & 1) : (hd & 3));
                const float tmx = __shfl_sync(0xffffffffu, mt[G >= 8 ? (hd >> 2) : 0], owner);
                mnew[hd] = fmaxf(m_run[hd], tmx);
                grow |= mnew[hd] > m_run[hd];
            }
            if (grow) {
                float al[G];
#pragma unroll
                for (int hd = 0; hd < G; hd++) {
                    al[hd] = (mnew[hd] == NEG_INF) ? 1.f : exp2f(m_run[hd] - mnew[hd]);
                    m_run[hd] = mnew[hd];
                }
#pragma unroll
                for (int hh = 0; hh < C::HPL; hh++) l_run[hh] *= pick<G>(al, lane_head<G>(c, hh));
#pragma unroll
                for (int i = 0; i < C::NTV; i++) {
                    const int col = 8 * i + (lane >> 2);
                    float f = 1.f;
#pragma unroll
                    for (int hd = 0; hd < G; hd++)
                        if (col % G == hd) f = al[hd];
                    Z[i] *= f;
                }
#pragma unroll
                for (int g = 0; g < 4; g++)
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        const int col = 8 * ((g * G) / 8) + 2 * c + (k & 1);
                        float f = 1.f;
#pragma unroll
                        for (int hd = 0; hd < G; hd++)
                            if (col % G == hd) f = al[hd];
                        O[2 * g][k] *= f;
                        O[2 * g + 1][k] *= f;
                    }
            }
#pragma unroll
            for (int bi = 0; bi < 2; bi++)
#pragma unroll
                for (int st = 0; st < 2; st++)
#pragma unroll
                    for (int hh = 0; hh < C::HPL; hh++) {
                        const float v = sco[bi][st][hh];
                        const float mm = pick<G>(m_run, lane_head<G>(c, hh));
                        const float p = (v == NEG_INF) ? 0.f : exp2f(v - mm);
                        P[bi][st][hh] = p;
                        l_run[hh] += p;
                    }
            // ---- P.V for my blocks
#pragma unroll
            for (int bi = 0; bi < 2; bi++) {
                if (bi < nmine) {
                    const uint8_t *blk = ring + s * STAGE_BYTES + (2 * warp + bi) * BLK_BYTES;
                    uint32_t Bv[C::NTV][2];
#pragma unroll
                    for (int i = 0; i < C::NTV; i++) {
                        const int col = 8 * i + (lane >> 2);
                        const bool valid = col < 4 * G;
                        const int gv = valid ? col / G : 0;
                        const int hv = col % G;
                        const int owner = G == 1 ? c : (G == 2 ? (hv & 1) : (hv & 3));
                        const int src0 = 4 * (2 * c) + owner, src1 = 4 * (2 * c + 1) + owner;
                        float pp[4];
#pragma unroll
                        for (int hh = 0; hh < C::HPL; hh++) {
                            const float q0 = __shfl_sync(0xffffffffu, P[bi][0][hh], src0);
                            const float q1 = __shfl_sync(0xffffffffu, P[bi][0][hh], src1);
                            const float q2 = __shfl_sync(0xffffffffu, P[bi][1][hh], src0);
                            const float q3 = __shfl_sync(0xffffffffu, P[bi][1][hh], src1);
                            if (hh == 0 || (hv >> 2) == hh) {
                                pp[0] = q0; pp[1] = q1; pp[2] = q2; pp[3] = q3;
                            }
                        }
                        const uint2 vsc = *reinterpret_cast<const uint2 *>(blk + OFF_VS + 8 * (4 * c + gv));
                        const uint2 vzr = *reinterpret_cast<const uint2 *>(blk + OFF_VZ + 8 * (4 * c + gv));
                        const float2 s01 = unpack_half2(vsc.x), s23 = unpack_half2(vsc.y);
                        const float2 z01 = unpack_half2(vzr.x), z23 = unpack_half2(vzr.y);
                        Bv[i][0] = valid ? pack_half2(pp[0] * s01.x, pp[1] * s01.y) : 0u;
                        Bv[i][1] = valid ? pack_half2(pp[2] * s23.x, pp[3] * s23.y) : 0u;
                        if (valid)
                            Z[i] += pp[0] * z01.x + pp[1] * z01.y + pp[2] * z23.x + pp[3] * z23.y;
                    }
                    const uint4 vq = *reinterpret_cast<const uint4 *>(blk + OFF_VC + 16 * (4 * r + c));
                    const uint32_t Wv[4] = {vq.x, vq.y, vq.z, vq.w};
#pragma unroll
                    for (int g = 0; g < 4; g++) {
                        const uint32_t msk = 0x00030003u << (2 * g);
                        const int nv = (g * G) / 8;
#pragma unroll
                        for (int h2 = 0; h2 < 2; h2++) {
                            const uint32_t w0 = Wv[h2], w2 = Wv[2 + h2];
                            mma16816(O[2 * g + h2], w0 & msk, (w0 >> 8) & msk, w2 & msk,
                                     (w2 >> 8) & msk, Bv[nv][0], Bv[nv][1]);
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        sc.cur += n;
        ++it;
        // end of this CTA's segment of the unit: write the partial
        if (sc.cur == sc.ustart + sc.nb || sc.cur == sc.end) {
            flush(blockIdx.x + unit);
            reset_state();
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Merge + rotate-out.
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128) decode_merge_kernel(DecodeArgs a) {
    __shared__ __align__(16) float o_s[D];
    const int hq = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int G = a.G, h = hq / G, head = hq % G;
    uint16_t *out = a.out + ((size_t)b * a.Hq + hq) * D;
    const int L = a.seq_lens[b];
    if (L < 1 || L > a.capacity) {
        out[t] = 0;
        return;
    }
    const int u = b * a.Hkv + h;
    const int nb = (a.prefix[b + 1] - a.prefix[b]) / a.Hkv;
    const int N = a.prefix[a.B];
    const int W = max(1, (N + a.C - 1) / a.C);
    const int ustart = a.prefix[b] + h * nb;
    int c0 = 0, c1 = -1;
    if (nb > 0) {
        c0 = ustart / W;
        c1 = (ustart + nb - 1) / W;
    }
    const float *sp = a.sinkp + ((size_t)b * a.Hq + hq) * PART;
    const bool has_sink = a.S > 0;
    float ms = has_sink ? sp[0] : NEG_INF;
    for (int cc = c0; cc <= c1; cc++)
        ms = fmaxf(ms, a.part[((size_t)(cc + u) * G + head) * PART]);
    float acc = 0.f, lsum = 0.f;
    if (has_sink && sp[0] != NEG_INF) {
        const float f = exp2f(sp[0] - ms);
        acc = f * sp[4 + t];
        lsum = f * sp[1];
    }
    for (int cc = c0; cc <= c1; cc++) {
        const float *pp = a.part + ((size_t)(cc + u) * G + head) * PART;
        const float f = exp2f(pp[0] - ms);
        acc = fmaf(f, pp[4 + t], acc);
        lsum = fmaf(f, pp[1], lsum);
    }
    o_s[t] = acc / lsum;
    __syncthreads();
    if (a.mode == KVQ_ROT_DENSE) {
        // out[i] = sum_j o[j] * R_v[h][i][j]: one warp per row, lanes over j
        const float *R = a.R_v + (size_t)h * D * D;
        const float4 o4 = *reinterpret_cast<const float4 *>(&o_s[4 * lane]);
        for (int i = warp; i < D; i += 4) {
            const float4 r4 = *reinterpret_cast<const float4 *>(R + (size_t)i * D + 4 * lane);
            float d = o4.x * r4.x + o4.y * r4.y + o4.z * r4.z + o4.w * r4.w;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
            if (lane == 0) out[i] = __half_as_ushort(__float2half_rn(d));
        }
    } else if (warp == 0) {
        float v[4] = {o_s[4 * lane], o_s[4 * lane + 1], o_s[4 * lane + 2], o_s[4 * lane + 3]};
        fwht128_warp(v);
        const int4 pi = *reinterpret_cast<const int4 *>(a.perm + ((size_t)a.Hkv + h) * D + 4 * lane);
        out[pi.x & (D - 1)] = __half_as_ushort(__float2half_rn(v[0] * 0.08838834764831845f));
        out[pi.y & (D - 1)] = __half_as_ushort(__float2half_rn(v[1] * 0.08838834764831845f));
        out[pi.z & (D - 1)] = __half_as_ushort(__float2half_rn(v[2] * 0.08838834764831845f));
        out[pi.w & (D - 1)] = __half_as_ushort(__float2half_rn(v[3] * 0.08838834764831845f));
    }
}

// ---------------------------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------------------------
size_t split_smem_bytes(int G) {
    return (size_t)NSTAGE * STAGE_BYTES + 2 * NSTAGE * sizeof(uint64_t) +
           sizeof(float) * (DEC_CONSUMER_WARPS * G * D + 2 * DEC_CONSUMER_WARPS * G +
                            DEC_CONSUMER_WARPS * G * 4) +
           16;
}

WsLayout ws_layout(int B, int Hq, int Hkv, int C) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    WsLayout w;
    const int G = Hq / Hkv;
    w.prefix = 0;
    w.qprep = up(w.prefix + sizeof(int32_t) * (B + 1));
    w.sinkp = up(w.qprep + sizeof(float) * (size_t)B * Hq * QP);
    w.part = up(w.sinkp + sizeof(float) * (size_t)B * Hq * PART);
    w.total = up(w.part + sizeof(float) * ((size_t)C + (size_t)B * Hkv) * G * PART);
    return w;
}

template <int G>
static cudaError_t launch_split(const DecodeArgs &a, cudaStream_t st) {
    const size_t smem = split_smem_bytes(G);
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<G>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_split_kernel<G><<<a.C, DEC_THREADS, smem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_decode(const uint16_t *Q, int Hq, const kvq_cache_desc &cd, int mode,
                          const float *R_k, const float *R_v, const int32_t *perm,
                          const int32_t *seq_lens, int C, void *ws, uint16_t *out,
                          cudaStream_t st) {
    const WsLayout w = ws_layout(cd.B, Hq, cd.Hkv, C);
    uint8_t *base = static_cast<uint8_t *>(ws);
    DecodeArgs a;
    a.Q = Q;
    a.blocks = static_cast<const uint8_t *>(cd.blocks);
    a.k_sink = cd.k_sink;
    a.v_sink = cd.v_sink;
    a.R_k = R_k;
    a.R_v = R_v;
    a.perm = perm;
    a.seq_lens = seq_lens;
    a.status = cd.status;
    a.prefix = reinterpret_cast<int32_t *>(base + w.prefix);
    a.qprep = reinterpret_cast<float *>(base + w.qprep);
    a.sinkp = reinterpret_cast<float *>(base + w.sinkp);
    a.part = reinterpret_cast<float *>(base + w.part);
    a.out = out;
    a.B = cd.B;
    a.Hq = Hq;
    a.Hkv = cd.Hkv;
    a.G = Hq / cd.Hkv;
    a.S = cd.sink_fp16;
    a.capacity = cd.capacity;
    a.nblk = cd.capacity / BLK_TOK;
    a.mode = mode;
    a.C = C;
    decode_prologue_kernel<<<dim3(Hq, cd.B), 128, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    switch (a.G) {
        case 1: e = launch_split<1>(a, st); break;
        case 2: e = launch_split<2>(a, st); break;
        case 4: e = launch_split<4>(a, st); break;
        case 8: e = launch_split<8>(a, st); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    decode_merge_kernel<<<dim3(Hq, cd.B), 128, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace kvq
