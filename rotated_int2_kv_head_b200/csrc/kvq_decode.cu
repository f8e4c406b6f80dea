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
// Three kernels per call:
//   decode_qprep_kernel     per (b, KV head): the G queries rotated by R_k
//                           (or perm + FWHT) and split into int8 hi/lo per
//                           group for the integer tensor cores.
//   decode_split_kernel<G>  stream-K over all cache blocks of all (b, h)
//                           units: every CTA takes an equal share of 16-token
//                           blocks (the schedule is derived from seq_lens by
//                           every CTA).  Thread 0 streams them into a
//                           shared-memory ring with 1-D bulk copies (TMA);
//                           four warps run the scores and P.V on tensor cores
//                           straight from the packed codes with an online
//                           softmax; each (CTA, unit) segment leaves one
//                           partial (m, l, o_rot[128]) per head.
//   decode_merge_kernel     per (b, query head): the sink partial (fp16 sinks,
//                           fp32 CUDA cores), the merge of all partials, then
//                           out = o_rot . R_v^T (or FWHT + inverse permutation).

// Tensor-core operand tricks.  Scores: a code byte masked with 0x03 << 2g is
// the u8 value c*4^g, so one AND turns 4 packed bytes into an m16n8k32 IMMA
// operand register; the query enters as an int8 hi/lo pair per group (about
// 15 bits) and the products accumulate exactly in int32.  P.V: a 2-bit code
// in bits [2g, 2g+1] of a 16-bit lane, every other bit zero, IS the fp16
// subnormal c*4^g*2^-24, so one AND gives an m16n8k16 HMMA operand register
// (two codes); the softmax weights times the fp16 V scales are the other
// operand.  The 4^g factors are folded into per-group fp32 scales.  The
// dequantisation c*s + z is factored: sum_j q_j (c_j s + z) =
// s*sum_j q_j c_j + z*sum_j q_j, so only the integer codes go through the MMA.
#include <atomic>

#include "kvq_internal.cuh"

namespace kvq {

// Split kernel: one CTA per SM made of DEC_GROUPS independent groups of
// GROUP_WARPS warps; each group streams its own ring of stages.
constexpr int DEC_GROUPS = 4;
constexpr int GROUP_WARPS = 4;
constexpr int GROUP_THREADS = 32 * GROUP_WARPS;           // 128
constexpr int DEC_THREADS = DEC_GROUPS * GROUP_THREADS;   // 512
constexpr int DEC_WARPS = DEC_GROUPS * GROUP_WARPS;       // 16
// Blocks per warp per stage and ring slots per group: four blocks (a 24 KB
// stage of 256 tokens, two in the ring) for G <= 4; two (12 KB, three in
// the ring) for G = 8, whose flush scratch leaves no room for 24 KB stages.
__host__ __device__ constexpr int bpw_for(int G) { return G >= 8 ? 2 : 4; }
__host__ __device__ constexpr int nstage_for(int G) { return G >= 8 ? 3 : 2; }
__host__ __device__ constexpr int stage_blks_for(int G) { return bpw_for(G) * GROUP_WARPS; }
__host__ __device__ constexpr int stage_bytes_for(int G) { return stage_blks_for(G) * BLK_BYTES; }
// Prepared query per query head, QB bytes:
//   int8 hi[128], int8 lo[128]  with q_s ~= sq_g * (hi + lo/254) per group g
//   float kap[4] = sq_g / 4^g,  float qsum[4] = sum of q_s over group g
constexpr int QB = 288;
constexpr int PART = 132;   // per partial: m, l, 0, 0, o[128]
constexpr float LOG2E = 1.4426950408889634f;
#define NEG_INF (__int_as_float(0xff800000))

struct DecodeArgs {
    const uint16_t *Q;
    const uint8_t *blocks;
    const int32_t *table;   // paged cache: [B][nblk] pool block per logical block, else null
    int num_blocks;         // paged: pool blocks
    const uint16_t *k_sink, *v_sink;
    const float *R_k, *R_v;
    const int32_t *perm;
    const int32_t *seq_lens;
    int32_t *status;
    uint8_t *qprep;    // [B*Hq][QB] prepared queries
    float *part;       // [(C+U)*G][PART]
    uint16_t *out;
    // S: leading fp16 sinks (positions 0..S-1; 0 with identified sinks).
    // Srows: fp16 sink rows per (b, h).  sink_pos / sink_count: identified
    // sinks ([B][Srows] ascending positions, rows in use), else null; their
    // INT2 slots carry a NaN K scale, so their scores come out NaN and are
    // turned into -inf.
    const int32_t *sink_pos, *sink_count;
    int Srows;
    int B, Hq, Hkv, G, S, capacity, nblk, mode, C;
    // qlen queries per sequence: query "head" hq (of Hq = heads x qlen) is
    // query i = hq % qlen of its head and sees positions < L - (qlen-1-i)
    int qlen;
    int out_rotated;   // 1: out = o_rot (the caller folds R_v^T into its projection)
    // KVLinC key correction adapter (or null): U, V fp32 [Hkv][128][adr]
    const float *adU, *adV;
    int adr;
};

// Blocks of 16 tokens that hold codes for a sequence of length L: positions
// [S, L) live in cache blocks S/16 .. (L-1)/16.
__device__ __forceinline__ int unit_blocks(int L, int S, int capacity) {
    if (L < 1 || L > capacity || L <= S) return 0;
    return (L - 1) / BLK_TOK - S / BLK_TOK + 1;
}

// Schedule slots of a unit: its blocks plus UNIT_PHANTOM leading phantom
// slots that stand for the cost of starting the unit (loading its queries,
// and the flush of the partial when a group leaves it; measured at about
// 8 blocks' streaming time).  Work is split evenly over slots, so a group
// whose range takes in the start of a unit streams that many fewer blocks
// and the groups finish together.  Phantom slots are skipped, never
// processed.
constexpr int UNIT_PHANTOM = 8;
__device__ __forceinline__ int unit_slots(int L, int S, int capacity) {
    const int nb = unit_blocks(L, S, capacity);
    return nb > 0 ? nb + UNIT_PHANTOM : 0;
}

// ---------------------------------------------------------------------------------------------
// Split kernel.
// ---------------------------------------------------------------------------------------------
// Per-CTA schedule over the global slot space: unit u = b*Hkv + h holds
// nb(b) = unit_slots consecutive slots (UNIT_PHANTOM phantom slots, then one
// per cache block) starting at prefix[b] + h*nb(b), where prefix[b] = Hkv *
// sum over b' < b of nb(b').  `pref` carries prefix[b].
struct Sched {
    int b, h, nb, ustart, cur, end, pref;
};

__device__ __forceinline__ int seq_blocks(const DecodeArgs &a, int b) {
    return unit_slots(a.seq_lens[b], a.S, a.capacity);
}

__device__ __forceinline__ void sched_fix_unit(Sched &s, const DecodeArgs &a) {
    // move (b, h) forward until cur lies inside the unit
    while (s.cur >= s.ustart + s.nb && s.cur < s.end) {
        if (++s.h == a.Hkv) {
            s.h = 0;
            s.pref += a.Hkv * s.nb;
            ++s.b;
            s.nb = seq_blocks(a, s.b);
        }
        s.ustart = s.pref + s.h * s.nb;
    }
}

// CTA-wide (all DEC_THREADS threads): total block count N from seq_lens, this
// CTA's range [c*W, min(N, (c+1)*W)) with W = ceil(N / C), split into
// DEC_GROUPS contiguous parts, and for each part the unit holding its first
// block: group g gets s (an empty range when the CTA's range is short).
// Thread t covers a contiguous run of sequences; an exclusive shuffle scan
// of the runs' block counts gives every run's offset.  scratch:
// 3*DEC_GROUPS + DEC_WARPS ints of shared memory.  Returns false when the
// CTA's range is empty (uniformly over the CTA).  CTA 0 flags invalid
// lengths.
constexpr int SCHED_SMALL_B = 32;
__device__ bool sched_init_cta(Sched &s, const DecodeArgs &a, int *scratch) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    if (a.B <= SCHED_SMALL_B) {
        // Few sequences: every thread reads all lengths (the same addresses
        // in every thread) and finds its group's first unit alone, with no
        // scan and no barrier.
        int N = 0;
#pragma unroll 4
        for (int b = 0; b < a.B; b++) {
            const int L = a.seq_lens[b];
            if (blockIdx.x == 0 && t == 0 && (L < 1 || L > a.capacity))
                set_status(a.status, KVQ_DEV_BAD_LEN);
            N += a.Hkv * unit_slots(L, a.S, a.capacity);
        }
        const int W = max(1, (N + a.C - 1) / a.C);
        const int beg = blockIdx.x * W, end = min(N, beg + W);
        if (beg >= end) return false;
        const int Wg = (end - beg + DEC_GROUPS - 1) / DEC_GROUPS;
        const int p = beg + (t / GROUP_THREADS) * Wg;
        s.b = s.h = s.nb = s.ustart = s.pref = 0;
        s.cur = s.end = 0;
        if (p < end) {
            int acc = 0;
            for (int b = 0; b < a.B; b++) {
                const int nbu = seq_blocks(a, b);
                if (p < acc + a.Hkv * nbu) {
                    s.b = b;
                    s.pref = acc;
                    s.nb = nbu;
                    break;
                }
                acc += a.Hkv * nbu;
            }
            s.h = (p - s.pref) / s.nb;
            s.ustart = s.pref + s.h * s.nb;
            s.cur = p;
            s.end = min(end, p + Wg);
        }
        return true;
    }
    const int per = (a.B + DEC_THREADS - 1) / DEC_THREADS;
    const int lo = min(a.B, t * per), hi = min(a.B, lo + per);
    int sum = 0, nb_lo = 0;          // nb_lo: blocks per unit of sequence lo (kept in a register)
    for (int b = lo; b < hi; b++) {
        const int L = a.seq_lens[b];
        if (blockIdx.x == 0 && (L < 1 || L > a.capacity)) set_status(a.status, KVQ_DEV_BAD_LEN);
        const int nb = unit_slots(L, a.S, a.capacity);
        if (b == lo) nb_lo = nb;
        sum += a.Hkv * nb;
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    int *wsum = scratch + 3 * DEC_GROUPS;         // [DEC_WARPS]
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int woff = 0, N = 0;
#pragma unroll
    for (int w2 = 0; w2 < DEC_WARPS; w2++) {
        const int v = wsum[w2];
        woff += (w2 < warp) ? v : 0;
        N += v;
    }
    const int cstart = woff + incl - sum, cend = woff + incl;   // this thread's run
    const int W = max(1, (N + a.C - 1) / a.C);
    const int beg = blockIdx.x * W, end = min(N, beg + W);
    if (beg >= end) return false;
    const int Wg = (end - beg + DEC_GROUPS - 1) / DEC_GROUPS;
    // the run holding each part's first block publishes (sequence, its first
    // global block, blocks per unit)
#pragma unroll
    for (int g = 0; g < DEC_GROUPS; g++) {
        const int p = beg + g * Wg;
        if (p < end && cstart <= p && p < cend) {
            int acc = cstart;
            for (int b = lo; b < hi; b++) {
                const int nbu = b == lo ? nb_lo : seq_blocks(a, b);
                if (p < acc + a.Hkv * nbu) {
                    scratch[3 * g] = b;
                    scratch[3 * g + 1] = acc;
                    scratch[3 * g + 2] = nbu;
                    break;
                }
                acc += a.Hkv * nbu;
            }
        }
    }
    __syncthreads();
    const int g = threadIdx.x / GROUP_THREADS;
    const int p = beg + g * Wg;
    if (p < end) {
        s.b = scratch[3 * g];
        s.pref = scratch[3 * g + 1];
        s.nb = scratch[3 * g + 2];
        s.h = (p - s.pref) / s.nb;
        s.ustart = s.pref + s.h * s.nb;
        s.cur = p;
        s.end = min(end, p + Wg);
    } else {
        s.b = s.h = s.nb = s.ustart = s.pref = 0;
        s.cur = s.end = 0;
    }
    return true;
}

// Next stage of a group's own range (up to max_blks blocks, never crossing
// a unit); false when the range is exhausted.  Leader thread only.
__device__ __forceinline__ bool sched_take(Sched &ps, const DecodeArgs &a, int max_blks, int &unit, int &b,
                                           int &h, int &kblk, int &n) {
    if (ps.cur >= ps.end) return false;
    sched_fix_unit(ps, a);
    const int first = ps.ustart + UNIT_PHANTOM;       // slot of the unit's block 0
    if (ps.cur < first) {                             // skip the phantom slots
        ps.cur = first;
        if (ps.cur >= ps.end) return false;
    }
    n = min(min(max_blks, ps.end - ps.cur), ps.ustart + ps.nb - ps.cur);
    unit = ps.b * a.Hkv + ps.h;
    b = ps.b;
    h = ps.h;
    kblk = ps.cur - first;
    ps.cur += n;
    return true;
}

// ---------------------------------------------------------------------------------------------
// Query preparation: per (b, KV head), the G queries rotated by R_k (or perm +
// FWHT), scaled by log2(e)/sqrt(128) so scores are exp2 exponents, and per
// group an int8 hi/lo pair on the scale max|q_s|/127 (about 15 significant
// bits): qprep[(b*Hq + hq)*QB] = {hi[128], lo[128], kap[4] = sq_g/4^g,
// qsum[4]}.  R_k (64 KB per head, the bulk of what it reads) is fetched
// before the dependency wait, alongside a preceding append; Q after it.
// ---------------------------------------------------------------------------------------------
// With a key correction adapter ("KVLinC : KV Cache Quantization with
// Hadamard Rotation and Linear Correction", abstract: lightweight linear
// adapters compensate for the errors of the quantized keys), every INT2 key
// k^ (model basis) is scored as k^ + (k^ . U) . V^T.  Its score against q is
// k^ . qc with qc = q + (q . V) . U^T, so the correction is folded into the
// query once per call: qc replaces q before the rotation, and the streaming
// kernel is unchanged.  The fp16 sinks (no quantization error) are scored by
// the merge kernel against the query as given.
constexpr int QP_THREADS = 256;

__global__ void __launch_bounds__(QP_THREADS) decode_qprep_kernel(DecodeArgs a) {
    __shared__ __align__(16) float red[QP_THREADS / 32][D];
    __shared__ __align__(16) float qr_s[D];
    __shared__ __align__(16) float qa_s[D], tv_s[D], qadj_s[D];   // adapter: q, q . V, qc
    const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int G = a.G;
    float4 rr[16];
    if (a.mode == KVQ_ROT_DENSE) {
        // warp w: rows 16w..16w+15 of R_k, lane l: columns 4l..4l+3, all loads in flight
        const float *R = a.R_k + (size_t)h * D * D + (size_t)(16 * warp) * D + 4 * lane;
#pragma unroll
        for (int ii = 0; ii < 16; ii++) rr[ii] = *reinterpret_cast<const float4 *>(R + ii * D);
    }
    // Waiting here (R_k is already on its way) and letting the split kernel
    // launch right away lets the query work below overlap its start-up.
    pdl_wait();
    pdl_trigger();
    // mark every split partial empty (m = -inf, l = 0): a group of the split
    // kernel writes only the units it took stages of
    {
        const size_t nslots = (size_t)DEC_GROUPS * ((size_t)a.C + (size_t)a.B * a.Hkv) * G;
        const size_t stride = (size_t)gridDim.x * gridDim.y * QP_THREADS;
        for (size_t i = ((size_t)blockIdx.y * gridDim.x + blockIdx.x) * QP_THREADS + t; i < nslots;
             i += stride)
            *reinterpret_cast<float2 *>(a.part + i * PART) = make_float2(NEG_INF, 0.f);
    }
    for (int hd = 0; hd < G; hd++) {
        const int hq = h * G + hd;
        const uint16_t *q = a.Q + ((size_t)b * a.Hq + hq) * D;
        __syncthreads();
        const bool adapt = a.adU != nullptr;
        if (adapt) {                                   // qc = q + (q . V) . U^T, fp32
            const float *U = a.adU + (size_t)h * D * a.adr, *V = a.adV + (size_t)h * D * a.adr;
            if (t < D) qa_s[t] = __half2float(__ushort_as_half(q[t]));
            __syncthreads();
            if (t < a.adr) {
                float acc = 0.f;
                for (int i = 0; i < D; i++) acc = fmaf(qa_s[i], V[(size_t)i * a.adr + t], acc);
                tv_s[t] = acc;
            }
            __syncthreads();
            if (t < D) {
                float acc = qa_s[t];
                for (int j = 0; j < a.adr; j++) acc = fmaf(U[(size_t)t * a.adr + j], tv_s[j], acc);
                qadj_s[t] = acc;
            }
            __syncthreads();
        }
        if (a.mode == KVQ_ROT_DENSE) {
            const uint4 u0 = *reinterpret_cast<const uint4 *>(q + 16 * warp);
            const uint4 u1 = *reinterpret_cast<const uint4 *>(q + 16 * warp + 8);
            const uint32_t w8[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int ii = 0; ii < 8; ii++) {
                const float2 x2 = adapt ? make_float2(qadj_s[16 * warp + 2 * ii],
                                                      qadj_s[16 * warp + 2 * ii + 1])
                                        : unpack_half2(w8[ii]);
                const float4 ra = rr[2 * ii], rb = rr[2 * ii + 1];
                acc.x = fmaf(x2.x, ra.x, acc.x); acc.y = fmaf(x2.x, ra.y, acc.y);
                acc.z = fmaf(x2.x, ra.z, acc.z); acc.w = fmaf(x2.x, ra.w, acc.w);
                acc.x = fmaf(x2.y, rb.x, acc.x); acc.y = fmaf(x2.y, rb.y, acc.y);
                acc.z = fmaf(x2.y, rb.z, acc.z); acc.w = fmaf(x2.y, rb.w, acc.w);
            }
            *reinterpret_cast<float4 *>(&red[warp][4 * lane]) = acc;
            __syncthreads();
            if (t < D) {
                float v = 0.f;
#pragma unroll
                for (int w2 = 0; w2 < QP_THREADS / 32; w2++) v += red[w2][t];
                qr_s[t] = v;
            }
        } else if (warp == 0) {
            const int4 pi = *reinterpret_cast<const int4 *>(a.perm + (size_t)h * D + 4 * lane);
            float v[4];
            if (adapt) {
                v[0] = qadj_s[pi.x & (D - 1)];
                v[1] = qadj_s[pi.y & (D - 1)];
                v[2] = qadj_s[pi.z & (D - 1)];
                v[3] = qadj_s[pi.w & (D - 1)];
            } else {
                v[0] = __half2float(__ushort_as_half(q[pi.x & (D - 1)]));
                v[1] = __half2float(__ushort_as_half(q[pi.y & (D - 1)]));
                v[2] = __half2float(__ushort_as_half(q[pi.z & (D - 1)]));
                v[3] = __half2float(__ushort_as_half(q[pi.w & (D - 1)]));
            }
            fwht128_warp(v);
            *reinterpret_cast<float4 *>(&qr_s[4 * lane]) =
                make_float4(v[0] * 0.08838834764831845f, v[1] * 0.08838834764831845f,
                            v[2] * 0.08838834764831845f, v[3] * 0.08838834764831845f);
        }
        __syncthreads();
        if (t < D) {
            // thread t = element t; warp g = group g
            const float qv = qr_s[t] * (LOG2E * 0.08838834764831845f);
            float gs = qv, amax = fabsf(qv);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                gs += __shfl_xor_sync(0xffffffffu, gs, off);
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            }
            const float sq = amax > 0.f ? amax * (1.0f / 127.0f) : 1.0f;
            const float u = qv / sq;
            const float hi = fminf(fmaxf(rintf(u), -127.f), 127.f);
            const float lo = fminf(fmaxf(rintf((u - hi) * 254.0f), -127.f), 127.f);
            uint8_t *qp = reinterpret_cast<uint8_t *>(a.qprep) + ((size_t)b * a.Hq + hq) * QB;
            qp[t] = (uint8_t)(int8_t)hi;
            qp[D + t] = (uint8_t)(int8_t)lo;
            if (lane == 0) {
                float *qf = reinterpret_cast<float *>(qp + 2 * D);
                qf[warp] = sq * __int_as_float((127 - 2 * warp) << 23);   // sq / 4^g
                qf[4 + warp] = gs;
            }
        }
    }
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

// Which (group, head) the score-layout lane with quad index c turns into
// P.V weights, for its k-th weight register (k < NW).
template <int G>
__device__ __forceinline__ void wsrc(int c, int k, int &g, int &head) {
    if (G == 1) { g = c; head = 0; }
    else if (G == 2) { g = (c >> 1) + 2 * k; head = c & 1; }
    else if (G == 4) { g = k; head = c; }
    else { g = k & 3; head = c + 4 * (k >> 2); }
}

// Shared-memory carve-out of the split kernel: DEC_GROUPS group regions of
// `gstride` bytes (ring, stage barriers, descriptors, flush scratch), then
// the schedule scratch.  Every piece starts on a
// 16-byte boundary (descriptors are read as int4, copies land 16-B aligned).
struct SplitSmem {
    unsigned full, desc, fo, fm, fl, fz, gstride, scratch, total;
};
__host__ __device__ constexpr unsigned smem_up16(unsigned x) { return (x + 15u) & ~15u; }
__host__ __device__ inline SplitSmem split_smem_layout(int G) {
    const unsigned ns = nstage_for(G);
    SplitSmem L{};
    L.full = ns * (unsigned)stage_bytes_for(G);                  // ring at offset 0
    L.desc = smem_up16(L.full + ns * 8u);
    L.fo = smem_up16(L.desc + 2u * ns * 16u);
    L.fm = smem_up16(L.fo + 4u * GROUP_WARPS * G * D);
    L.fl = smem_up16(L.fm + 4u * GROUP_WARPS * G);
    L.fz = smem_up16(L.fl + 4u * GROUP_WARPS * G);
    L.gstride = (L.fz + 4u * GROUP_WARPS * G * 4 + 4u + 127u) & ~127u;   // + one dump float
    L.scratch = DEC_GROUPS * L.gstride;
    L.total = smem_up16(L.scratch + 4u * (3 * DEC_GROUPS + DEC_WARPS));
    return L;
}

// Index of the partial a group writes for a unit: (CTA, unit) pairs of a
// static contiguous split never collide under c + u, and each has one slot
// per group.
__host__ __device__ inline size_t part_slot(int cta, int unit, int grp) {
    return (size_t)DEC_GROUPS * ((size_t)cta + unit) + grp;
}

template <int G, bool PAGED>
__global__ void __launch_bounds__(DEC_THREADS, 1) decode_split_kernel(DecodeArgs a) {
    using C = Cfg<G>;
    constexpr int NS = nstage_for(G);
    constexpr int BPW = bpw_for(G);
    constexpr int STAGE_BLKS = stage_blks_for(G);
    constexpr int STAGE_BYTES = stage_bytes_for(G);
    constexpr int NW = G;                              // weight registers per lane per block
    constexpr int NGL = G == 1 ? 1 : (G == 2 ? 2 : 4); // V-meta groups a lane reads
    extern __shared__ __align__(128) uint8_t smem[];
    const SplitSmem L = split_smem_layout(G);
    const int grp = threadIdx.x / GROUP_THREADS, gt = threadIdx.x % GROUP_THREADS;
    const int warp = gt >> 5, lane = threadIdx.x & 31;        // warp within the group
    const bool leader = gt == 0;
    uint8_t *gbase = smem + grp * L.gstride;
    uint8_t *ring = gbase;                                            // [NS][STAGE_BYTES]
    uint64_t *full = reinterpret_cast<uint64_t *>(gbase + L.full);    // [NS]
    int4 *desc = reinterpret_cast<int4 *>(gbase + L.desc);            // [2*NS] stage descriptors
    float *fo = reinterpret_cast<float *>(gbase + L.fo);              // [W][G][128]
    float *fm = reinterpret_cast<float *>(gbase + L.fm);              // [W][G]
    float *fl = reinterpret_cast<float *>(gbase + L.fl);              // [W][G]
    float *fz = reinterpret_cast<float *>(gbase + L.fz);              // [W][G][4]
    float *dump = fz + GROUP_WARPS * G * 4;                           // write-only
    int *scratch = reinterpret_cast<int *>(smem + L.scratch);
    // named barrier of this group (id 0 is __syncthreads)
    auto bar_group = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "n"(GROUP_THREADS) : "memory"); };

    if (leader) {
        for (int k = 0; k < NS; k++) mbar_init(&full[k], 1);
        fence_mbar_init();
    }
    __syncthreads();
    // The append before this decode has completed (the query-preparation
    // kernel waited on it before letting this kernel launch), so seq_lens and
    // the cache are read - and the first copies issued - before waiting on
    // the prepared queries.
    Sched sc;   // this group's part of the CTA's range (warp 0's copy is the producer state)
    if (!sched_init_cta(sc, a, scratch)) {
        pdl_wait();
        pdl_trigger();
        return;
    }
    const int fb = a.S / BLK_TOK;

    // Copies.  Ring slot `slot` is filled with the next stage of the group's
    // range, with its descriptor {unit, b, h, first cache block}, {n}; unit -1
    // marks the end (the slot's phase is completed by a plain arrive).
    // Descriptors are written at least one group barrier before anyone
    // reads them, so they are read without waiting on the copy.
    // Producer: the group leader for a contiguous cache (a stage is one bulk
    // copy); the group's whole first warp for a paged one, all lanes in step
    // (the schedule state sc evolves identically in every lane), lane j
    // copying block j of the stage so that the table entries load in
    // parallel.  Lane 0 writes the descriptor and the expected byte count.
    int issued = 0;      // stages issued (= the iteration they belong to)
    bool ended = false;  // the end marker is written
    auto issue_next = [&](int slot) {
        if (ended) return;
        int unit = 0, b = 0, h = 0, kblk = 0, n = 0;
        if (sched_take(sc, a, STAGE_BLKS, unit, b, h, kblk, n)) {
            if (lane == 0) {
                desc[2 * slot] = make_int4(unit, b, h, fb + kblk);
                desc[2 * slot + 1] = make_int4(n, 0, 0, 0);
                mbar_arrive_expect_tx(&full[slot], n * BLK_BYTES);
            }
            if (!PAGED) {          // contiguous: the stage's blocks are adjacent
                if (lane == 0)
                    bulk_g2s(ring + slot * STAGE_BYTES,
                             a.blocks + ((size_t)unit * a.nblk + fb + kblk) * (size_t)BLK_BYTES,
                             n * BLK_BYTES, &full[slot]);
            } else if (lane < n) { // paged: block `lane` of the stage
                const int ph = a.table[(size_t)b * a.nblk + fb + kblk + lane];
                const bool okb = ph >= 0 && ph < a.num_blocks;
                if (!okb) set_status(a.status, KVQ_DEV_BAD_TABLE);
                const size_t bi = okb ? (size_t)ph * a.Hkv + h : 0;   // bad entry: block 0
                bulk_g2s(ring + slot * STAGE_BYTES + lane * BLK_BYTES, a.blocks + bi * BLK_BYTES,
                         BLK_BYTES, &full[slot]);
            }
        } else {
            if (lane == 0) {
                desc[2 * slot] = make_int4(-1, 0, 0, 0);
                mbar_arrive(&full[slot]);
            }
            ended = true;
        }
        ++issued;
    };
    const bool producer = PAGED ? warp == 0 : leader;   // contiguous: lane 0 alone suffices
    // A range of 3 to 8 stages (short contexts, where the start is a large
    // part of the kernel) issues its first stage alone and the rest of the
    // ring once that stage has landed: when every group asks for its whole
    // ring at once, the copies issued last land over 2 us after the first
    // (llama7b: 29 MB at once) and those groups also finish last.  With two
    // stages the second one's later copy would end the range later; G <= 2
    // only: the G = 4 and 8 kernels have no registers to spare for it.
    const int span = sc.end - sc.cur;
    const bool staged = G <= 2 && span > 2 * STAGE_BLKS && span <= 8 * STAGE_BLKS;
    if (producer)
        for (int k = 0; k < (staged ? 1 : NS); k++) issue_next(k);
    bar_group();
    pdl_wait();
    pdl_trigger();

    const int r = lane >> 2, c = lane & 3;
    // per-unit query operands
    uint32_t qB[4][C::NTK_STEP][2];
    float qsum[C::NTK], kap2[C::NTK];
    int Lcur = 0;
    // online-softmax state; m_lane[hh] = m_run of the head this lane's
    // scores in slot hh belong to (refreshed when the maxima move)
    float m_run[G], m_lane[C::HPL], l_run[C::HPL], O[8][4], Z[NW];
    int cur_unit = -1;

    auto reset_state = [&]() {
#pragma unroll
        for (int i = 0; i < G; i++) m_run[i] = NEG_INF;
#pragma unroll
        for (int i = 0; i < C::HPL; i++) {
            l_run[i] = 0.f;
            m_lane[i] = NEG_INF;
        }
#pragma unroll
        for (int i = 0; i < 8; i++)
#pragma unroll
            for (int k = 0; k < 4; k++) O[i][k] = 0.f;
#pragma unroll
        for (int i = 0; i < NW; i++) Z[i] = 0.f;
    };

    auto load_unit = [&](int b, int h) {
        // B fragments of the K-side IMMA, one per group: column n of the N
        // tile is (group, head, hi/lo); k = element e of the group
        const uint8_t *qbase = a.qprep + ((size_t)b * a.Hq + (size_t)h * G) * QB;
        const int n = lane >> 2;
#pragma unroll
        for (int g = 0; g < 4; g++) {
#pragma unroll
            for (int j = 0; j < C::NTK_STEP; j++) {
                const int nu = (g * 2 * G) / 8 + j;
                const int col = 8 * nu + n;
                const int gcol = col / (2 * G), head = (col % (2 * G)) / 2, hl = col & 1;
                uint32_t b0 = 0u, b1 = 0u;
                if (gcol == g) {
                    const uint8_t *qh = qbase + head * QB + hl * D + 32 * g;
                    b0 = *reinterpret_cast<const uint32_t *>(qh + 4 * c);
                    b1 = *reinterpret_cast<const uint32_t *>(qh + 16 + 4 * c);
                }
                qB[g][j][0] = b0;
                qB[g][j][1] = b1;
            }
        }
#pragma unroll
        for (int nu = 0; nu < C::NTK; nu++) {
            const int g = ktile_group<G>(nu, c), head = ktile_head<G>(nu, c);
            const float *qf = reinterpret_cast<const float *>(qbase + head * QB + 2 * D);
            kap2[nu] = qf[g] * (1.0f / 254.0f);
            qsum[nu] = qf[4 + g];
        }
        Lcur = a.seq_lens[b];
    };

    auto flush = [&](int slot) {
        // reduce l and Z over the 8 row lanes
#pragma unroll
        for (int i = 0; i < C::HPL; i++) {
            l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 4);
            l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 8);
            l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 16);
        }
#pragma unroll
        for (int i = 0; i < NW; i++) {
            Z[i] += __shfl_xor_sync(0xffffffffu, Z[i], 4);
            Z[i] += __shfl_xor_sync(0xffffffffu, Z[i], 8);
            Z[i] += __shfl_xor_sync(0xffffffffu, Z[i], 16);
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
#pragma unroll
            for (int k = 0; k < NW; k++) {
                int g, head;
                wsrc<G>(lane, k, g, head);
                fz[(warp * G + head) * 4 + g] = Z[k];
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
                    const int head = col % G;
                    const int j = 32 * g + 16 * h2 + 2 * r + (k >> 1);
                    const float val = O[g * 2 + h2][k] * __int_as_float((127 + 24 - 2 * g) << 23);
                    if constexpr (G >= 4) {
                        // an accumulator of another group's column goes to the
                        // dump float: with a branch on the lane here the compiler
                        // kept O in local memory (a 16-byte store per stage)
                        float *dst = col / G == g ? &wo[head * D + j] : dump;
                        *dst = val;
                    } else if (col / G == g) {
                        wo[head * D + j] = val;
                    }
                }
        bar_group();
        const int tj = gt;            // 0..127: element
        for (int head = 0; head < G; head++) {
            float ms = NEG_INF;
#pragma unroll
            for (int w = 0; w < GROUP_WARPS; w++) ms = fmaxf(ms, fm[w * G + head]);
            float acc = 0.f, lsum = 0.f;
#pragma unroll
            for (int w = 0; w < GROUP_WARPS; w++) {
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
        bar_group();
    };

    // Scores, part 1: the K codes of blocks b_lo .. b_hi-1 of the warp's
    // BPW blocks of a stage through the integer tensor cores (one IMMA per
    // group and block; blocks past the stage's end are masked later).
    auto k_mma = [&](const uint8_t *blk0, int (&dk)[BPW][C::NTK][4], int b_lo, int b_hi) {
        uint4 kq[BPW];
#pragma unroll
        for (int bi = b_lo; bi < b_hi; bi++)
            kq[bi] = *reinterpret_cast<const uint4 *>(blk0 + bi * BLK_BYTES + 16 * (4 * r + c));
        // one IMMA per group: the masked bytes are u8 codes c * 4^g.  The
        // first group feeding an N tile starts its accumulator from zero.
#pragma unroll
        for (int g = 0; g < 4; g++) {
            const uint32_t msk = 0x03030303u << (2 * g);
            const bool first = g == 0 || (g * 2 * G) / 8 != ((g - 1) * 2 * G) / 8;
#pragma unroll
            for (int bi = b_lo; bi < b_hi; bi++) {
                const uint4 q4 = kq[bi];
#pragma unroll
                for (int j = 0; j < C::NTK_STEP; j++) {
                    const int nu = (g * 2 * G) / 8 + j;
                    if (first)
                        imma16832_zc(dk[bi][nu], q4.x & msk, q4.z & msk, q4.y & msk, q4.w & msk,
                                     qB[g][j][0], qB[g][j][1]);
                    else
                        imma16832(dk[bi][nu], q4.x & msk, q4.z & msk, q4.y & msk, q4.w & msk,
                                  qB[g][j][0], qB[g][j][1]);
                }
            }
        }
    };
    // Scores, part 2: integer dots -> fp32 scores (group scale and zero,
    // query scale), summed over the groups; positions outside [S, L) and
    // phantom blocks are masked to -inf.  A plain stage (every block of the
    // warp's share real and inside [S, L), no identified sinks in the cache)
    // needs neither the masks nor the NaN guard; PLAIN is a constant at
    // each inlined call.
    auto k_combine = [&](const bool PLAIN, const uint8_t *blk0, const int (&dk)[BPW][C::NTK][4],
                         int tok0, int nmine, float (&sco)[BPW][2][C::HPL], bool (&edge)[BPW],
                         int b_lo, int b_hi) {
        // a block needs masking if it is a phantom or crosses [S, L)
#pragma unroll
        for (int bi = b_lo; bi < b_hi; bi++)
            edge[bi] = !PLAIN && (bi >= nmine || tok0 + bi * BLK_TOK < a.S ||
                                  tok0 + (bi + 1) * BLK_TOK > Lcur - (a.qlen - 1));
#pragma unroll
        for (int bi = b_lo; bi < b_hi; bi++) {
            float part_sc[2][C::HPL];
#pragma unroll
            for (int st = 0; st < 2; st++)
#pragma unroll
                for (int hh = 0; hh < C::HPL; hh++) part_sc[st][hh] = 0.f;
            // the K-side N tiles of one group share the tokens' scale / zero:
            // one tile per group for G <= 4, the group's two head halves for G = 8
            constexpr int TPG = G >= 8 ? 2 : 1;
#pragma unroll
            for (int gi = 0; gi < C::NTK / TPG; gi++) {
                const int g = ktile_group<G>(gi * TPG, c);
                const uint2 mk = *reinterpret_cast<const uint2 *>(blk0 + bi * BLK_BYTES + OFF_KM +
                                                                  8 * (4 * r + g));
                const float2 sz0 = unpack_half2(mk.x), sz1 = unpack_half2(mk.y);
#pragma unroll
                for (int j = 0; j < TPG; j++) {
                    const int nu = gi * TPG + j;
                    const int hh = ktile_slot<G>(nu);
                    // hi*254 + lo is exact in int32 (|.| < 2^28)
                    const float d0 = __int2float_rn(dk[bi][nu][0] * 254 + dk[bi][nu][1]) * kap2[nu];
                    const float d1 = __int2float_rn(dk[bi][nu][2] * 254 + dk[bi][nu][3]) * kap2[nu];
                    part_sc[0][hh] = fmaf(sz0.x, d0, fmaf(sz0.y, qsum[nu], part_sc[0][hh]));
                    part_sc[1][hh] = fmaf(sz1.x, d1, fmaf(sz1.y, qsum[nu], part_sc[1][hh]));
                }
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
                    if (edge[bi]) {
                        const int pos = tok0 + bi * BLK_TOK + r + 8 * st;
                        const int lim = Lcur - (a.qlen - 1 - lane_head<G>(c, hh) % a.qlen);
                        v = (bi < nmine && pos >= a.S && pos < lim) ? v : NEG_INF;
                    }
                    // an identified sink's slot scores NaN (its K scale is the
                    // marker): fmax with -inf returns -inf for NaN, v otherwise
                    sco[bi][st][hh] = PLAIN ? v : fmaxf(v, NEG_INF);
                }
        }
    };
    // Online softmax and P.V of one stage.
    auto v_side = [&](const uint8_t *blk0, const float (&sco)[BPW][2][C::HPL], const bool (&edge)[BPW]) {
        // ---- online softmax.  The running max only moves when a score of
        // this stage exceeds it (rare after the first stages), so the
        // common path is one vote; the branch is uniform over the warp.
        bool over = false;
#pragma unroll
        for (int bi = 0; bi < BPW; bi++)
#pragma unroll
            for (int st = 0; st < 2; st++)
#pragma unroll
                for (int hh = 0; hh < C::HPL; hh++)
                    over |= sco[bi][st][hh] > m_lane[hh];
        if (__any_sync(0xffffffffu, over)) {
        float mt[C::HPL];
#pragma unroll
        for (int hh = 0; hh < C::HPL; hh++) {
            float v = NEG_INF;
#pragma unroll
            for (int bi = 0; bi < BPW; bi++) v = fmaxf(v, fmaxf(sco[bi][0][hh], sco[bi][1][hh]));
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
            mt[hh] = v;
        }
        float mnew[G];
        bool grow = false;
#pragma unroll
        for (int hd = 0; hd < G; hd++) {
            const int owner = G == 1 ? 0 : (G == 2 ? (hd & 1) : (hd & 3));
            const float tmx = __shfl_sync(0xffffffffu, mt[G >= 8 ? (hd >> 2) : 0], owner);
            mnew[hd] = fmaxf(m_run[hd], tmx);
            grow |= mnew[hd] > m_run[hd];
        }
        if (grow) {
            float al[G];
#pragma unroll
            for (int hd = 0; hd < G; hd++) {
                al[hd] = (mnew[hd] == NEG_INF) ? 1.f : fast_exp2(m_run[hd] - mnew[hd]);
                m_run[hd] = mnew[hd];
            }
#pragma unroll
            for (int hh = 0; hh < C::HPL; hh++) m_lane[hh] = pick<G>(m_run, lane_head<G>(c, hh));
#pragma unroll
            for (int hh = 0; hh < C::HPL; hh++) l_run[hh] *= pick<G>(al, lane_head<G>(c, hh));
#pragma unroll
            for (int k = 0; k < NW; k++) {
                int g, head;
                wsrc<G>(c, k, g, head);
                Z[k] *= pick<G>(al, head);
            }
#pragma unroll
            for (int g = 0; g < 4; g++)
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const int col = 8 * ((g * G) / 8) + 2 * c + (k & 1);
                    const float f = pick<G>(al, col % G);
                    O[2 * g][k] *= f;
                    O[2 * g + 1][k] *= f;
                }
        }
        }
        float P[BPW][2][C::HPL];
#pragma unroll
        for (int bi = 0; bi < BPW; bi++)
#pragma unroll
            for (int st = 0; st < 2; st++)
#pragma unroll
                for (int hh = 0; hh < C::HPL; hh++) {
                    const float v = sco[bi][st][hh];
                    const float mr = m_lane[hh];
                    // a masked score (-inf) must give exactly 0: with several
                    // queries per sequence a head can have seen no valid
                    // position yet (mr = -inf), so subtract 0 then
                    const float mm = mr == NEG_INF ? 0.f : mr;
                    const float p = fast_exp2(v - mm);
                    P[bi][st][hh] = p;
                    l_run[hh] += p;
                }
        // ---- P.V
#pragma unroll
        for (int bi = 0; bi < BPW; bi++) {
            const uint8_t *blk = blk0 + bi * BLK_BYTES;
            // weights w = p * s_v in the score layout, as half2 (token r, token r+8):
            // p packed to fp16 times the two tokens' fp16 scales (one HMUL2)
            uint32_t H[NW];
            {
                uint32_t spair[NGL];
                float zr[NGL][2];
#pragma unroll
                for (int gl = 0; gl < NGL; gl++) {
                    const int g = G == 1 ? c : (G == 2 ? (c >> 1) + 2 * gl : gl);
                    const uint2 mv = *reinterpret_cast<const uint2 *>(blk + OFF_VM + 8 * (4 * r + g));
                    spair[gl] = __byte_perm(mv.x, mv.y, 0x5410);      // (s_r, s_r+8)
                    zr[gl][0] = __half2float(__ushort_as_half((unsigned short)(mv.x >> 16)));
                    zr[gl][1] = __half2float(__ushort_as_half((unsigned short)(mv.y >> 16)));
                }
#pragma unroll
                for (int k = 0; k < NW; k++) {
                    const int gl = G == 1 ? 0 : (G == 2 ? k : (k & 3));
                    const int hh = G >= 8 ? (k >> 2) : 0;
                    const float p0 = P[bi][0][hh], p1 = P[bi][1][hh];
                    const uint32_t ph = pack_half2(p0, p1);
                    const __half2 w2 = __hmul2(*reinterpret_cast<const __half2 *>(&ph),
                                               *reinterpret_cast<const __half2 *>(&spair[gl]));
                    uint32_t hw = *reinterpret_cast<const uint32_t *>(&w2);
                    float z0 = zr[gl][0], z1 = zr[gl][1];
                    if (edge[bi]) {      // masked tokens (p == 0): never use their metadata
                        hw &= (p0 == 0.f ? 0xffff0000u : 0xffffffffu) &
                              (p1 == 0.f ? 0x0000ffffu : 0xffffffffu);
                        z0 = p0 == 0.f ? 0.f : z0;
                        z1 = p1 == 0.f ? 0.f : z1;
                    }
                    H[k] = hw;
                    Z[k] = fmaf(p0, z0, fmaf(p1, z1, Z[k]));
                }
            }
            // B fragments: lane (n, c') needs tokens 2c', 2c'+1, 2c'+8, 2c'+9 of
            // its column (group, head)
            uint32_t Bv[C::NTV][2];
#pragma unroll
            for (int i = 0; i < C::NTV; i++) {
                const int col = 8 * i + (lane >> 2);
                const bool valid = col < 4 * G;
                const int g = col / G, head = col % G;
                int csrc, ksel;
                if (G == 1) { csrc = g; ksel = 0; }
                else if (G == 2) { csrc = head + 2 * (g & 1); ksel = g >> 1; }
                else if (G == 4) { csrc = head; ksel = g & 1; }
                else { csrc = head & 3; ksel = head >> 2; }
                const int src0 = 4 * (2 * c) + csrc, src1 = src0 + 4;
                uint32_t X, Y;
                if (G == 1) {
                    X = __shfl_sync(0xffffffffu, H[0], src0);
                    Y = __shfl_sync(0xffffffffu, H[0], src1);
                } else {
                    // two candidate registers; the lane keeps the one it needs
                    const int k0 = G == 2 ? 0 : (G == 4 ? 2 * i : i);
                    const int k1 = G == 2 ? 1 : (G == 4 ? 2 * i + 1 : 4 + i);
                    const uint32_t X0 = __shfl_sync(0xffffffffu, H[k0], src0);
                    const uint32_t Y0 = __shfl_sync(0xffffffffu, H[k0], src1);
                    const uint32_t X1 = __shfl_sync(0xffffffffu, H[k1], src0);
                    const uint32_t Y1 = __shfl_sync(0xffffffffu, H[k1], src1);
                    X = ksel ? X1 : X0;
                    Y = ksel ? Y1 : Y0;
                }
                Bv[i][0] = valid ? __byte_perm(X, Y, 0x5410) : 0u;
                Bv[i][1] = valid ? __byte_perm(X, Y, 0x7632) : 0u;
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
                    mma16816(O[2 * g + h2], w0 & msk, (w0 >> 8) & msk, w2 & msk, (w2 >> 8) & msk,
                             Bv[nv][0], Bv[nv][1]);
                }
            }
        }
    };
    // Release ring slot `slot` once the whole group is done with it; the
    // group's first warp refills it.  Returns true (uniformly over the group) when a wait
    // failed anywhere in the group: the group then stops.
    auto release = [&](int slot, bool ok) -> bool {
        int any_bad;
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %1, 0;\n\t"
            "bar.red.or.pred p, %2, %3, p;\n\tselp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(any_bad)
            : "r"((unsigned)!ok), "r"(1 + grp), "n"(GROUP_THREADS)
            : "memory");
        if (any_bad) return true;
        if (producer) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue_next(slot);
        }
        return false;
    };
    auto wblk = [&](int slot) { return ring + slot * STAGE_BYTES + (BPW * warp) * BLK_BYTES; };

    reset_state();
    if (staged) {
        // staged start, before the loop so that the loop is the same for
        // every range: the first unit's queries, then (producer) the rest of
        // the ring once stage 0 has landed.  After a failed wait it stays
        // unissued; the loop's own wait then fails and the group drains.
        const int4 d0 = desc[0];
        if (d0.x >= 0) {
            load_unit(d0.y, d0.z);
            cur_unit = d0.x;
        }
        if (producer && mbar_wait_bounded(&full[0], 0))
            for (int k = 1; k < NS; k++) issue_next(k);
    }
    bool aborted = false;
    int it = 0;
    for (;; ++it) {
        const int s = it % NS;
        const int4 d0 = desc[2 * s];
        const int n = desc[2 * s + 1].x;
        const int unit = d0.x;
        if (unit < 0) break;                               // end of the schedule
        if (unit != cur_unit) {                            // uniform over the group
            if (cur_unit >= 0) {
                flush(part_slot(blockIdx.x, cur_unit, grp));
                reset_state();
            }
            load_unit(d0.y, d0.z);
            cur_unit = unit;
        }
        const bool ok = mbar_wait_bounded(&full[s], (it / NS) & 1);
        const int nmine = min(BPW, max(0, n - BPW * warp));
        if (ok && nmine > 0) {
            int dk[BPW][C::NTK][4];
            float sco[BPW][2][C::HPL];
            bool edge[BPW];
            const int tok0 = (d0.w + BPW * warp) * BLK_TOK;
            // the K side in pairs of blocks; one block at a time where the
            // integer accumulators of two do not fit the registers: G = 8, and
            // G = 4 on a contiguous cache, whose interior-stage copy then spills
            // nothing (56 bytes with pairs; gqa_sinks 191.5 -> 187.4 us)
            constexpr int KSTEP = (G >= 8 || (G == 4 && !PAGED)) ? 1 : 2;
            auto stage_body = [&](const bool PLAIN) {
#pragma unroll
                for (int b0 = 0; b0 < BPW; b0 += KSTEP) {
                    k_mma(wblk(s), dk, b0, b0 + KSTEP);
                    k_combine(PLAIN, wblk(s), dk, tok0, nmine, sco, edge, b0, b0 + KSTEP);
                }
                v_side(wblk(s), sco, edge);
            };
            // uniform over the warp: all BPW blocks real, inside [S, L - qlen + 1),
            // and no identified-sink markers possible.  Not for G = 8: its second
            // copy of the stage body spills enough to cost what it saves.
            const bool plain = G <= 4 && !a.sink_pos && nmine == BPW && tok0 >= a.S &&
                               tok0 + BPW * BLK_TOK <= Lcur - (a.qlen - 1);
            if (plain)
                stage_body(true);
            else
                stage_body(false);
        }
        if (!ok) set_status(a.status, KVQ_DEV_TIMEOUT);
        if (release(s, ok)) {
            aborted = true;
            break;
        }
    }
    if (aborted) {
        // leave no copy in flight into this CTA's shared memory: wait (with
        // the full bound) for every stage issued from this iteration on
        if (leader) drain_ring(full, NS, it, issued);
        return;
    }
    if (cur_unit >= 0) flush(part_slot(blockIdx.x, cur_unit, grp));
}

// ---------------------------------------------------------------------------------------------
// Merge + rotate-out.
// ---------------------------------------------------------------------------------------------
constexpr int MRG_THREADS = 256;
constexpr int MRG_BATCH = 32;     // partials loaded together

__global__ void __launch_bounds__(MRG_THREADS) decode_merge_kernel(DecodeArgs a) {
    __shared__ __align__(16) float o_s[D];
    __shared__ __align__(16) float red[MRG_THREADS / 32][D];
    __shared__ float wred[MRG_THREADS / 32];
    __shared__ int ired[2 * (MRG_THREADS / 32)];
    __shared__ __align__(16) float qs[D];
    __shared__ float ssc[MAX_SINK];
    __shared__ __align__(16) float sinkp[PART];          // the sink partial: m, l, 0, 0, o[128]
    const int hq = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
    const int warp = t >> 5, lane = t & 31;
    const int G = a.G, h = hq / G, head = hq % G;
    uint16_t *out = a.out + ((size_t)b * a.Hq + hq) * D;
    // Before waiting on the split kernel: only data that kernel does not write
    // (its predecessor, the append, has completed by the time this kernel can
    // start).  The sink partial, in fp32 on CUDA cores: q_rot, scores over the
    // fp16 sink rows, softmax, weighted sum.
    const int L = a.seq_lens[b];
    const int Li = L - (a.qlen - 1 - hq % a.qlen);           // this query's context
    const bool lok = (L >= 1 && L <= a.capacity && Li >= 1);
    // fp16 rows this query sees: rows 0..ns-1.  Leading sinks: positions
    // < min(S, Li).  Identified sinks: the listed positions below Li (a
    // prefix of the ascending list).
    int ns;
    if (!a.sink_pos) {
        ns = (a.S > 0 && lok) ? min(a.S, Li) : 0;
    } else {
        const int n = min(max(a.sink_count[b], 0), a.Srows);
        ns = __syncthreads_count(lok && t < n && a.sink_pos[(size_t)b * a.Srows + t] < Li);
    }
    if (ns > 0) {
        const uint16_t *q = a.Q + ((size_t)b * a.Hq + hq) * D;
        if (a.mode == KVQ_ROT_DENSE) {
            const float *R = a.R_k + (size_t)h * D * D + (size_t)(16 * warp) * D + 4 * lane;
            float4 rr[16];
#pragma unroll
            for (int ii = 0; ii < 16; ii++) rr[ii] = *reinterpret_cast<const float4 *>(R + ii * D);
            const uint4 u0 = *reinterpret_cast<const uint4 *>(q + 16 * warp);
            const uint4 u1 = *reinterpret_cast<const uint4 *>(q + 16 * warp + 8);
            const uint32_t w8[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int ii = 0; ii < 8; ii++) {
                const float2 x2 = unpack_half2(w8[ii]);
                const float4 ra = rr[2 * ii], rb = rr[2 * ii + 1];
                acc.x = fmaf(x2.x, ra.x, acc.x); acc.y = fmaf(x2.x, ra.y, acc.y);
                acc.z = fmaf(x2.x, ra.z, acc.z); acc.w = fmaf(x2.x, ra.w, acc.w);
                acc.x = fmaf(x2.y, rb.x, acc.x); acc.y = fmaf(x2.y, rb.y, acc.y);
                acc.z = fmaf(x2.y, rb.z, acc.z); acc.w = fmaf(x2.y, rb.w, acc.w);
            }
            *reinterpret_cast<float4 *>(&red[warp][4 * lane]) = acc;
            __syncthreads();
            if (t < D) {
                float v = 0.f;
#pragma unroll
                for (int w2 = 0; w2 < MRG_THREADS / 32; w2++) v += red[w2][t];
                qs[t] = v;
            }
        } else if (warp == 0) {
            const int4 pi = *reinterpret_cast<const int4 *>(a.perm + (size_t)h * D + 4 * lane);
            float v[4] = {__half2float(__ushort_as_half(q[pi.x & (D - 1)])),
                          __half2float(__ushort_as_half(q[pi.y & (D - 1)])),
                          __half2float(__ushort_as_half(q[pi.z & (D - 1)])),
                          __half2float(__ushort_as_half(q[pi.w & (D - 1)]))};
            fwht128_warp(v);
            *reinterpret_cast<float4 *>(&qs[4 * lane]) =
                make_float4(v[0] * 0.08838834764831845f, v[1] * 0.08838834764831845f,
                            v[2] * 0.08838834764831845f, v[3] * 0.08838834764831845f);
        }
        __syncthreads();
        if (t < D) qs[t] *= LOG2E * 0.08838834764831845f;      // exp2 domain, like the partials
        __syncthreads();
        const uint16_t *ks = a.k_sink + ((size_t)b * a.Hkv + h) * a.Srows * D;
        const uint16_t *vs = a.v_sink + ((size_t)b * a.Hkv + h) * a.Srows * D;
        for (int tk = warp; tk < ns; tk += MRG_THREADS / 32) {
            const uint2 uu = *reinterpret_cast<const uint2 *>(ks + (size_t)tk * D + 4 * lane);
            const float2 k01 = unpack_half2(uu.x), k23 = unpack_half2(uu.y);
            float d = qs[4 * lane] * k01.x + qs[4 * lane + 1] * k01.y + qs[4 * lane + 2] * k23.x +
                      qs[4 * lane + 3] * k23.y;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
            if (lane == 0) ssc[tk] = d;
        }
        __syncthreads();
        if (t < D) {
            float m = NEG_INF;
            for (int tk = 0; tk < ns; tk++) m = fmaxf(m, ssc[tk]);
            float l = 0.f, o = 0.f;
            for (int tk = 0; tk < ns; tk++) {
                const float p = exp2f(ssc[tk] - m);
                l += p;
                o = fmaf(p, __half2float(__ushort_as_half(vs[(size_t)tk * D + t])), o);
            }
            sinkp[4 + t] = o;
            if (t == 0) {
                sinkp[0] = m;
                sinkp[1] = l;
            }
        }
        __syncthreads();
    }
    // This unit's place in the split kernel's block list, from seq_lens (the
    // same arithmetic the split CTAs use): blocks of sequences before b, and
    // in total.
    {
        int sb = 0, sn = 0;
        for (int i = t; i < a.B; i += MRG_THREADS) {
            const int nbi = a.Hkv * unit_slots(a.seq_lens[i], a.S, a.capacity);
            sn += nbi;
            sb += i < b ? nbi : 0;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            sb += __shfl_xor_sync(0xffffffffu, sb, off);
            sn += __shfl_xor_sync(0xffffffffu, sn, off);
        }
        if (lane == 0) {
            ired[warp] = sb;
            ired[MRG_THREADS / 32 + warp] = sn;
        }
    }
    // R_v rows for the rotate-out (no kernel of this chain writes R_v): warp w
    // rows 16w..16w+15, lane l columns 4l..4l+3, each load one whole row
    float4 rr[16];
    if (a.mode == KVQ_ROT_DENSE) {
        const float *R = a.R_v + (size_t)h * D * D + (size_t)(16 * warp) * D + 4 * lane;
#pragma unroll
        for (int ii = 0; ii < 16; ii++) rr[ii] = *reinterpret_cast<const float4 *>(R + ii * D);
    }
    __syncthreads();
    int pre = 0, N = 0;
#pragma unroll
    for (int w2 = 0; w2 < MRG_THREADS / 32; w2++) {
        pre += ired[w2];
        N += ired[MRG_THREADS / 32 + w2];
    }
    pdl_wait();
    pdl_trigger();
    if (!lok) {
        if (t < D) out[t] = 0;
        if (t == 0 && L >= 1 && L <= a.capacity) set_status(a.status, KVQ_DEV_BAD_LEN);   // L < qlen
        return;
    }
    const int u = b * a.Hkv + h;
    const int nb = unit_slots(L, a.S, a.capacity);
    const int W = max(1, (N + a.C - 1) / a.C);
    const int ustart = pre + h * nb;
    const int c0 = nb > 0 ? ustart / W : 0;
    const int np = nb > 0 ? (ustart + nb - 1) / W - c0 + 1 : 0;
    // partial i < DEC_GROUPS*np: group i % DEC_GROUPS of CTA c0 + i / DEC_GROUPS
    // (m = -inf if that group took no stage of the unit); then the sink partial
    auto pptr = [&](int i) -> const float * {
        return i < DEC_GROUPS * np
                   ? a.part + (part_slot(c0 + i / DEC_GROUPS, u, i % DEC_GROUPS) * G + head) * PART
                   : sinkp;
    };
    const int ntot = DEC_GROUPS * np + (ns > 0 ? 1 : 0);

    // Partials in batches of MRG_BATCH: warp w takes partials w, w+8, w+16,
    // w+24 of the batch and issues all their loads before using any.
    constexpr int PW = MRG_BATCH / (MRG_THREADS / 32);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.f, mglob = NEG_INF;
    for (int base = 0; base < ntot; base += MRG_BATCH) {
        float2 ml[PW];
        float4 o4[PW];
#pragma unroll
        for (int j = 0; j < PW; j++) {
            const int i = base + warp + j * (MRG_THREADS / 32);
            if (i < ntot) {
                const float *pp = pptr(i);
                ml[j] = make_float2(pp[0], pp[1]);
                o4[j] = *reinterpret_cast<const float4 *>(pp + 4 + 4 * lane);
            } else {
                ml[j] = make_float2(NEG_INF, 0.f);
                o4[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        float mloc = NEG_INF;
#pragma unroll
        for (int j = 0; j < PW; j++) mloc = fmaxf(mloc, ml[j].x);
        if (lane == 0) wred[warp] = mloc;
        __syncthreads();
        float mnew = mglob;
#pragma unroll
        for (int w2 = 0; w2 < MRG_THREADS / 32; w2++) mnew = fmaxf(mnew, wred[w2]);
        __syncthreads();
        const float fold = (mglob == NEG_INF) ? 0.f : exp2f(mglob - mnew);
        acc.x *= fold; acc.y *= fold; acc.z *= fold; acc.w *= fold;
        lsum *= fold;
        mglob = mnew;
#pragma unroll
        for (int j = 0; j < PW; j++) {
            // an empty partial (m = -inf) has only its header written: its
            // o and l are skipped, never multiplied by 0
            if (ml[j].x == NEG_INF) continue;
            const float f = exp2f(ml[j].x - mglob);
            acc.x = fmaf(f, o4[j].x, acc.x); acc.y = fmaf(f, o4[j].y, acc.y);
            acc.z = fmaf(f, o4[j].z, acc.z); acc.w = fmaf(f, o4[j].w, acc.w);
            lsum = fmaf(f, ml[j].y, lsum);
        }
    }
    *reinterpret_cast<float4 *>(&red[warp][4 * lane]) = acc;
    if (lane == 0) wred[warp] = lsum;
    __syncthreads();
    if (t < D) {
        float v = 0.f, l = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < MRG_THREADS / 32; w2++) {
            v += red[w2][t];
            l += wred[w2];
        }
        o_s[t] = v / l;
    }
    __syncthreads();
    if (a.out_rotated) {
        // the caller folds R_v^T into its own projection: o_rot as it is
        if (t < D) out[t] = __half_as_ushort(__float2half_rn(o_s[t]));
    } else if (a.mode == KVQ_ROT_DENSE) {
        // out[i] = sum_j o[j] R_v[h][i][j] for the warp's 16 rows: each lane
        // dots its 4 columns, then a reduce-scatter over the lanes (at the
        // exchange over lane bit m a lane keeps the half of its rows that bit
        // selects) leaves row 8b4 + 4b3 + 2b2 + b1 of lane bits b4..b1 in
        // lanes 2k and 2k+1: 16 shuffles instead of 5 per row
        const float4 o4 = *reinterpret_cast<const float4 *>(&o_s[4 * lane]);
        float v[16];
#pragma unroll
        for (int ii = 0; ii < 16; ii++)
            v[ii] = o4.x * rr[ii].x + o4.y * rr[ii].y + o4.z * rr[ii].z + o4.w * rr[ii].w;
#pragma unroll
        for (int m = 16, n = 8; m >= 2; m >>= 1, n >>= 1) {
            const bool up = (lane & m) != 0;
#pragma unroll
            for (int i = 0; i < n; i++) {
                const float send = up ? v[i] : v[i + n];
                const float keep = up ? v[i + n] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
        }
        const float d = v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
        const int row = 8 * ((lane >> 4) & 1) + 4 * ((lane >> 3) & 1) + 2 * ((lane >> 2) & 1) +
                        ((lane >> 1) & 1);
        if ((lane & 1) == 0) out[16 * warp + row] = __half_as_ushort(__float2half_rn(d));
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
    static_assert(sizeof(Sched) <= 32, "producer state slot");
    return split_smem_layout(G).total;
}

WsLayout ws_layout(int B, int Hq, int Hkv, int C) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    WsLayout w;
    const int G = Hq / Hkv;
    w.qprep = 0;
    w.part = up(w.qprep + (size_t)B * Hq * QB);
    w.total = up(w.part + sizeof(float) * DEC_GROUPS * ((size_t)C + (size_t)B * Hkv) * G * PART);
    return w;
}

template <int G, bool PAGED>
static cudaError_t launch_split_t(const DecodeArgs &a, cudaStream_t st) {
    const size_t smem = split_smem_bytes(G);
    // the dynamic shared-memory opt-in holds per device: set it once on each
    static std::atomic<unsigned long long> opted{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = (dev >= 0 && dev < 64) ? 1ull << dev : 0ull;
    if (bit == 0ull || (opted.load(std::memory_order_acquire) & bit) == 0ull) {
        e = cudaFuncSetAttribute(decode_split_kernel<G, PAGED>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        opted.fetch_or(bit, std::memory_order_acq_rel);
    }
    return launch_pdl(decode_split_kernel<G, PAGED>, dim3(a.C), dim3(DEC_THREADS), smem, st, a);
}

template <int G>
static cudaError_t launch_split(const DecodeArgs &a, cudaStream_t st) {
    return a.table ? launch_split_t<G, true>(a, st) : launch_split_t<G, false>(a, st);
}

cudaError_t launch_decode(const uint16_t *Q, int Hq, const kvq_cache_desc &cd, int mode,
                          const float *R_k, const float *R_v, const int32_t *perm,
                          const int32_t *seq_lens, int C, void *ws, uint16_t *out,
                          cudaStream_t st, cudaEvent_t ev_begin, cudaEvent_t ev_end, int qlen,
                          int out_rotated, const KeyAdapter &ad) {
    const WsLayout w = ws_layout(cd.B, Hq, cd.Hkv, C);
    uint8_t *base = static_cast<uint8_t *>(ws);
    DecodeArgs a;
    a.Q = Q;
    a.blocks = static_cast<const uint8_t *>(cd.blocks);
    a.table = cd.block_table;
    a.num_blocks = cd.num_blocks;
    a.k_sink = cd.k_sink;
    a.v_sink = cd.v_sink;
    a.R_k = R_k;
    a.R_v = R_v;
    a.perm = perm;
    a.seq_lens = seq_lens;
    a.status = cd.status;
    a.qprep = base + w.qprep;
    a.part = reinterpret_cast<float *>(base + w.part);
    a.out = out;
    a.B = cd.B;
    a.Hq = Hq;
    a.Hkv = cd.Hkv;
    a.G = Hq / cd.Hkv;
    a.sink_pos = cd.sink_pos;
    a.sink_count = cd.sink_count;
    a.Srows = cd.sink_fp16;
    a.S = cd.sink_pos ? 0 : cd.sink_fp16;
    a.capacity = cd.capacity;
    a.nblk = cd.capacity / BLK_TOK;
    a.mode = mode;
    a.C = C;
    a.qlen = qlen;
    a.out_rotated = out_rotated;
    a.adU = ad.U;
    a.adV = ad.V;
    a.adr = ad.r;
    cudaError_t e = launch_pdl(decode_qprep_kernel, dim3(cd.Hkv, cd.B), dim3(QP_THREADS), 0, st, a);
    if (e != cudaSuccess) return e;
    if (ev_begin && (e = cudaEventRecord(ev_begin, st)) != cudaSuccess) return e;
    switch (a.G) {
        case 1: e = launch_split<1>(a, st); break;
        case 2: e = launch_split<2>(a, st); break;
        case 4: e = launch_split<4>(a, st); break;
        case 8: e = launch_split<8>(a, st); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    if (ev_end && (e = cudaEventRecord(ev_end, st)) != cudaSuccess) return e;
    return launch_pdl(decode_merge_kernel, dim3(Hq, cd.B), dim3(MRG_THREADS), 0, st, a);
}

// ---------------------------------------------------------------------------------------------
// Test kernel for the give-up path of the bounded waits.  One thread runs the
// split kernel's ring protocol on a two-slot ring: stage 0 is a real 1536-byte
// bulk copy of `src`; slot 1 is never filled (a flag nothing sets), so the
// wait on it runs out after poll_limit polls.  The thread then flags
// KVQ_DEV_TIMEOUT and drains the ring with drain_ring - the same call the
// split kernel makes before an aborted CTA returns - and reports:
//   result[0] = 1 if the wait on the empty slot gave up, result[1] = stages
//   drain_ring could not see land (0 expected), result[2] = the sum of the
//   copied bytes as they sit in shared memory (the copy landed before the
//   CTA returned).
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(32) debug_wait_timeout_kernel(const uint8_t *src,
                                                                 uint32_t poll_limit,
                                                                 int32_t *status, int32_t *result) {
    __shared__ __align__(128) uint8_t ring[2][BLK_BYTES];
    __shared__ __align__(8) uint64_t full[2];
    if (threadIdx.x != 0) return;
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&full[0], BLK_BYTES);
    bulk_g2s(ring[0], src, BLK_BYTES, &full[0]);
    const int issued = 1;                       // slot 1: nothing is ever issued
    const bool ok = mbar_wait_bounded(&full[1], 0u, poll_limit);
    if (!ok) set_status(status, KVQ_DEV_TIMEOUT);
    const int lost = drain_ring(full, 2, 0, issued);
    int sum = 0;
    for (int i = 0; i < BLK_BYTES; i++) sum += ring[0][i];
    result[0] = ok ? 0 : 1;
    result[1] = lost;
    result[2] = sum;
}

cudaError_t launch_debug_wait_timeout(const uint8_t *src, uint32_t poll_limit, int32_t *status,
                                      int32_t *result, cudaStream_t st) {
    debug_wait_timeout_kernel<<<1, 32, 0, st>>>(src, poll_limit, status, result);
    return cudaGetLastError();
}

}  // namespace kvq
