// Decode attention over a cache whose keys were rotated before RoPE, across
// groups of GH consecutive KV heads ("RotateKV: Accurate and Robust 2-Bit KV
// Cache Quantization for LLMs via Outlier-Aware Adaptive Rotations", abstract
// item (ii)).  The cached key of position t is the quantized slice of
// FWHT_n(k_group[perm]) / sqrt(n), n = 128*GH, so the attention key is
//   k_t = RoPE_t( (FWHT_n(k_hat_group) / sqrt(n)) scattered through perm )
// for the head's slice: every position needs its own inverse rotation and
// its own RoPE angle, which no single query-side transform can absorb.  The
// values are rotated per head as in FWHT mode and the rotation is removed
// once, after the attention.
//
// Split kernels (one per group shape) and a merge kernel:
//   prerope_split_q_kernel  GH = G = 1 (below): four positions per warp step.
//   prerope_split_kernel<GH, G>  every other shape; grid (splits, B * Hkv/GH).  A CTA of 8 warps
//       takes a contiguous range of 16-token cache blocks of one (b, group),
//       split into 8 equal token runs, one per warp, taken in order.  Per
//       token: the GH heads' K codes are dequantised (4 elements
//       per lane), un-rotated by a warp FWHT (stages over the lane's 4
//       elements and the 32 lanes by shuffles, stages across the GH heads in
//       registers), scattered back through the permutation in shared memory,
//       RoPE'd (the pair partner of channel c < 64 is c + 64, 16 lanes away)
//       and dotted with each query head; online softmax and P.V on the
//       dequantised rotated values.  Each CTA leaves one partial
//       (m, l, o_rot[128]) per query head.
//   prerope_merge_kernel  per (b, query head): the partial over the fp16
//       sinks ("RotateKV", item (iii); keys kept pre-RoPE and turned at their
//       positions), the merge of all partials, and the removal of the value
//       rotation (FWHT + inverse permutation).
// The RoPE angle t * theta_f is taken as 2 pi * frac(t * theta_f / (2 pi))
// in fp64 at a warp's first token in every 16-token block (theta_f / (2 pi) comes from
// the host in fp64), then advanced token by token with the rotation by
// theta_f, so fp32 never holds an angle larger than 2 pi.
#include "kvq_internal.cuh"

namespace kvq {

constexpr int PR_WARPS = 8;
constexpr int PR_THREADS = 32 * PR_WARPS;
constexpr int PR_PART = 132;           // m, l, 0, 0, o[128]
constexpr int PR_MIN_BLOCKS = 8;       // cache blocks per split at least
constexpr float PR_LOG2E = 1.4426950408889634f;
#define PR_NEG_INF (__int_as_float(0xff800000))
// Start of a running max: finite, below any score, so exp2(score - max) is
// never exp2(-inf - -inf); a run without tokens keeps it with l = 0, o = 0,
// which every merge weights by exp2(PR_M0 - max) = 0 (or carries as zeros).
constexpr float PR_M0 = -1.0e30f;

// The four 2-bit codes of a lane (bits 2*g4 of the bytes of w) as exact
// floats: each byte is put under the exponent of 2^23 and 2^23 subtracted.
__device__ __forceinline__ void unpack4(uint32_t w, int g4, float c[4]) {
    const uint32_t m = (w >> (2 * g4)) & 0x03030303u;
#pragma unroll
    for (int k = 0; k < 4; k++)
        c[k] = __uint_as_float(__byte_perm(m, 0x4B000000u, 0x7540u + k)) - 8388608.0f;
}

struct PreRopeArgs {
    const uint16_t *Q;          // [B][Hq][128] post-RoPE queries
    const uint8_t *blocks;
    const int32_t *table;       // paged cache, else null
    int num_blocks;
    const int32_t *perm;        // [2][Hkv*128]: key groups, then value heads
    const int32_t *seq_lens;
    int32_t *status;
    float *part;                // [B*Hq][nsplit][PR_PART]
    uint16_t *out;              // [B][Hq][128]
    // fp16 sinks: rows [B][Hkv][Srows][128] (keys pre-RoPE as given, values
    // rotated); leading sinks are positions < S, identified ones listed in
    // sink_pos [B][Srows] (sink_count rows in use) with a NaN-marked INT2 slot
    const uint16_t *k_sink, *v_sink;
    const int32_t *sink_pos, *sink_count;
    int S, Srows;
    int B, Hq, Hkv, capacity, nblk, nsplit, bps;
    double phi[D / 2];          // theta_f / (2 pi), theta_f = base^(-2f/128)
};

// Splits per (b, group): 12 CTAs per SM in all, i.e. whole waves at 1, 2, 3,
// 4 or 6 resident CTAs per SM (equal ranges, so waves end together), and
// at least PR_MIN_BLOCKS cache blocks per split.
__host__ __device__ inline int pr_nsplit(int B, int ngroups, int max_ctx, int sms) {
    const int nb = (max_ctx + BLK_TOK - 1) / BLK_TOK;
    const int units = B * ngroups;
    int want = (12 * sms) / units;
    const int most = (nb + PR_MIN_BLOCKS - 1) / PR_MIN_BLOCKS;
    if (want > most) want = most;
    return want < 1 ? 1 : want;
}

template <int GH, int G>
__global__ void __launch_bounds__(PR_THREADS) prerope_split_kernel(PreRopeArgs a) {
    constexpr int n = GH * D;
    constexpr int NQ = GH * G;                        // query heads of the group
    __shared__ __align__(16) int32_t pg_s[n];         // the group's key permutation
    // per warp: the un-rotation scatter (n floats), then the warp's o (NQ x 128)
    __shared__ __align__(16) float kb_s[PR_WARPS][NQ * D];
    __shared__ float m_s[PR_WARPS][NQ], l_s[PR_WARPS][NQ];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int ng = a.Hkv / GH;
    const int b = blockIdx.y / ng, grp = blockIdx.y % ng;
    const float isq = GH == 1 ? 0.08838834764831845f
                              : (GH == 2 ? 0.0625f : (GH == 4 ? 0.04419417382415922f : 0.03125f));
    pdl_wait();
    pdl_trigger();
    for (int i = threadIdx.x; i < n; i += PR_THREADS)
        pg_s[i] = a.perm[(size_t)grp * n + i] & (n - 1);
    const int L = a.seq_lens[b];
    const bool lok = L >= 1 && L <= a.capacity;
    const int nb = lok ? (L + BLK_TOK - 1) / BLK_TOK : 0;
    const int blk0 = split * a.bps, blk1 = min(nb, blk0 + a.bps);

    // queries of the group, in the exp2 domain with the 1/sqrt(128) scale
    float qr[NQ][4];
#pragma unroll
    for (int i = 0; i < NQ; i++) {
        const int hq = grp * NQ + i;       // = (grp*GH + j)*G + g
        const uint2 u = *reinterpret_cast<const uint2 *>(a.Q + ((size_t)b * a.Hq + hq) * D + 4 * lane);
        const float2 x01 = unpack_half2(u.x), x23 = unpack_half2(u.y);
        const float sc = PR_LOG2E * 0.08838834764831845f;
        qr[i][0] = x01.x * sc;
        qr[i][1] = x01.y * sc;
        qr[i][2] = x23.x * sc;
        qr[i][3] = x23.y * sc;
    }
    // RoPE frequencies of the lane's 4 channels (f = (4 lane + k) mod 64):
    // the per-token step rotation
    float cst[4], snt[4];
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const int f = 4 * (lane & 15) + k;
        sincospif((float)(2.0 * a.phi[f]), &snt[k], &cst[k]);
    }
    const float psign = lane < 16 ? -1.f : 1.f;       // c < 64: x cos - x' sin

    float m_run[NQ], l_run[NQ], o[NQ][4];
#pragma unroll
    for (int i = 0; i < NQ; i++) {
        m_run[i] = PR_M0;
        l_run[i] = 0.f;
#pragma unroll
        for (int k = 0; k < 4; k++) o[i][k] = 0.f;
    }
    __syncthreads();                                  // pg_s
    int4 preg[GH <= 2 ? GH : 1];                      // small groups: the lane's indices in registers
#pragma unroll
    for (int j = 0; j < (GH <= 2 ? GH : 1); j++)
        preg[j] = *reinterpret_cast<const int4 *>(&pg_s[j * D + 4 * lane]);

    const int wi = lane & 7, g4 = lane >> 3;          // logical code word, quant group
    // the CTA's tokens in PR_WARPS contiguous, equal runs, one per warp
    // (leading sinks are not INT2 tokens: they start at S)
    const int t_beg = min(L, max(a.S, blk0 * BLK_TOK)), t_end = max(t_beg, min(L, blk1 * BLK_TOK));
    const int per = (t_end - t_beg + PR_WARPS - 1) / PR_WARPS;
    const int w0 = min(t_end, t_beg + warp * per), w1 = min(t_end, w0 + per);
    for (int blk = w0 / BLK_TOK; w0 < w1 && blk <= (w1 - 1) / BLK_TOK; blk++) {
        // block addresses of the group's GH heads (and the V block of each)
        const uint8_t *bp[GH];
#pragma unroll
        for (int j = 0; j < GH; j++) {
            const long long bi = cache_block_index(a.table, a.num_blocks, a.nblk, a.Hkv, b,
                                                   grp * GH + j, blk);
            if (bi < 0 && lane == 0) set_status(a.status, KVQ_DEV_BAD_TABLE);
            bp[j] = a.blocks + (size_t)(bi < 0 ? 0 : bi) * BLK_BYTES;
        }
        // the warp's next block into L2 while this one is worked on (its
        // 1536-byte blocks are 12 lines per head)
        if ((blk + 1) * BLK_TOK < w1 && lane < 12) {
#pragma unroll
            for (int j = 0; j < GH; j++) {
                const long long bn = cache_block_index(a.table, a.num_blocks, a.nblk, a.Hkv, b,
                                                       grp * GH + j, blk + 1);
                if (bn >= 0)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(a.blocks + (size_t)bn * BLK_BYTES +
                                                                  128 * lane));
            }
        }
        const int tau0 = max(w0, blk * BLK_TOK) - blk * BLK_TOK;
        const int tau1 = min(w1, (blk + 1) * BLK_TOK) - blk * BLK_TOK;
        // RoPE angle of the first token taken here, reduced in fp64
        float cs[4], sn[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const double u = (double)(blk * BLK_TOK + tau0) * a.phi[4 * (lane & 15) + k];
            const double fr = u - floor(u);
            sincospif((float)(2.0 * fr), &sn[k], &cs[k]);
        }
        for (int tau = tau0; tau < tau1; tau++) {
            const int r = tau & 7, th = tau >> 3;
            float v[GH][4];
#pragma unroll
            for (int j = 0; j < GH; j++) {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(
                    bp[j] + 16 * (4 * r + (wi & 3)) + 4 * (2 * th + (wi >> 2)));
                const uint32_t mk =
                    *reinterpret_cast<const uint32_t *>(bp[j] + 1024 + 8 * (4 * r + g4) + 4 * th);
                const float2 sz = unpack_half2(mk);
                const float s = sz.x * isq, z = sz.y * isq;
                float cf[4];
                unpack4(w, g4, cf);
#pragma unroll
                for (int k = 0; k < 4; k++) v[j][k] = fmaf(cf[k], s, z);
                fwht128_warp(v[j]);
            }
#pragma unroll
            for (int st = 1; st < GH; st <<= 1)
#pragma unroll
                for (int j = 0; j < GH; j++)
                    if ((j & st) == 0)
#pragma unroll
                        for (int k = 0; k < 4; k++) {
                            const float x0 = v[j][k], x1 = v[j + st][k];
                            v[j][k] = x0 + x1;
                            v[j + st][k] = x0 - x1;
                        }
            // k_pre[perm[i]] = y[i]: scatter, then read back in channel order
#pragma unroll
            for (int j = 0; j < GH; j++) {
                const int4 pi = GH <= 2 ? preg[j] : *reinterpret_cast<const int4 *>(&pg_s[j * D + 4 * lane]);
                kb_s[warp][pi.x] = v[j][0];
                kb_s[warp][pi.y] = v[j][1];
                kb_s[warp][pi.z] = v[j][2];
                kb_s[warp][pi.w] = v[j][3];
            }
            __syncwarp();
#pragma unroll
            for (int j = 0; j < GH; j++) {
                const float4 x = *reinterpret_cast<const float4 *>(&kb_s[warp][j * D + 4 * lane]);
                v[j][0] = x.x;
                v[j][1] = x.y;
                v[j][2] = x.z;
                v[j][3] = x.w;
            }
            __syncwarp();
            // RoPE at position t: channel c < 64 with its partner c + 64
#pragma unroll
            for (int j = 0; j < GH; j++)
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const float px = __shfl_xor_sync(0xffffffffu, v[j][k], 16);
                    v[j][k] = fmaf(psign * px, sn[k], v[j][k] * cs[k]);
                }
#pragma unroll
            for (int j = 0; j < GH; j++) {
                // rotated values of head j at this token: pieces 2wi, 2wi+1
                const int q2 = tau >> 1, side = tau & 1;
                const uint8_t *vb = bp[j] + 512;
                const int w0 = 2 * wi, w1 = 2 * wi + 1;
                const uint32_t c0 = *reinterpret_cast<const uint16_t *>(
                    vb + 16 * (4 * (w0 & 7) + (q2 & 3)) + 4 * (2 * (q2 >> 2) + (w0 >> 3)) + 2 * side);
                const uint32_t c1 = *reinterpret_cast<const uint16_t *>(
                    vb + 16 * (4 * (w1 & 7) + (q2 & 3)) + 4 * (2 * (q2 >> 2) + (w1 >> 3)) + 2 * side);
                const uint32_t vw = c0 | (c1 << 16);
                const uint32_t vmk =
                    *reinterpret_cast<const uint32_t *>(bp[j] + 1280 + 8 * (4 * r + g4) + 4 * th);
                const float2 vsz = unpack_half2(vmk);
                float vv[4];
                unpack4(vw, g4, vv);
#pragma unroll
                for (int k = 0; k < 4; k++) vv[k] = fmaf(vv[k], vsz.x, vsz.y);
#pragma unroll
                for (int g = 0; g < G; g++) {
                    const int i = j * G + g;
                    float d = qr[i][0] * v[j][0] + qr[i][1] * v[j][1] + qr[i][2] * v[j][2] +
                              qr[i][3] * v[j][3];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
                    // an identified sink's slot (NaN scale) scores NaN: fmax with
                    // -inf makes it -inf, whose weight below is exp2(-inf) = 0
                    // (m_run starts at PR_M0, finite)
                    d = fmaxf(d, PR_NEG_INF);
                    if (d > m_run[i]) {
                        const float al = exp2f(m_run[i] - d);   // 0 for the first token
                        l_run[i] *= al;
#pragma unroll
                        for (int k = 0; k < 4; k++) o[i][k] *= al;
                        m_run[i] = d;
                    }
                    const float p = exp2f(d - m_run[i]);
                    l_run[i] += p;
#pragma unroll
                    for (int k = 0; k < 4; k++) o[i][k] = fmaf(p, vv[k], o[i][k]);
                }
            }
            // next token: turn the RoPE angle by theta_f
#pragma unroll
            for (int k = 0; k < 4; k++) {
                const float c2 = cs[k] * cst[k] - sn[k] * snt[k];
                sn[k] = fmaf(sn[k], cst[k], cs[k] * snt[k]);
                cs[k] = c2;
            }
        }
    }

    // combine the warps through kb_s, reused as [PR_WARPS][NQ][128]
    __syncthreads();
    float *ob = &kb_s[0][0];
#pragma unroll
    for (int i = 0; i < NQ; i++) {
        *reinterpret_cast<float4 *>(&ob[((size_t)warp * NQ + i) * D + 4 * lane]) =
            make_float4(o[i][0], o[i][1], o[i][2], o[i][3]);
        if (lane == 0) {
            m_s[warp][i] = m_run[i];
            l_s[warp][i] = l_run[i];
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < NQ * D; e += PR_THREADS) {
        const int i = e / D, c = e % D;
        float mx = PR_NEG_INF;
#pragma unroll
        for (int w = 0; w < PR_WARPS; w++) mx = fmaxf(mx, m_s[w][i]);
        float lt = 0.f, ot = 0.f;
        if (mx != PR_NEG_INF) {
#pragma unroll
            for (int w = 0; w < PR_WARPS; w++) {
                if (m_s[w][i] == PR_NEG_INF) continue;        // a warp without tokens
                const float f = exp2f(m_s[w][i] - mx);
                lt = fmaf(f, l_s[w][i], lt);
                ot = fmaf(f, ob[((size_t)w * NQ + i) * D + c], ot);
            }
        }
        const int hq = grp * NQ + i;
        float *pp = a.part + (((size_t)b * a.Hq + hq) * a.nsplit + split) * PR_PART;
        pp[4 + c] = ot;
        if (c == 0) {
            pp[0] = mx;
            pp[1] = lt;
        }
    }
}

// ---- one KV head per group and one query per KV head (gh = G = 1) --------------------------
// The same CTA ranges, warp runs and partials as prerope_split_kernel, but a
// warp step takes four positions at once, eight lanes per position: lane
// (p, j) = (lane >> 3, lane & 7) holds, of position tb + p, the elements
// e = 32g + 4j + k (g, k < 4) of the stored (rotated) key and value, which
// in the block layout are logical code word j: one 4-byte load per row.
// The FWHT's index bits 0, 1 (k) and 5, 6 (g) are butterflies inside the
// lane, bits 2, 3, 4 (j) across the position's eight lanes.  The
// un-rotated key goes through shared memory in channel order (the
// permutation scatter), and lane j takes back channels 8j..8j+7 and their
// RoPE partners 64+8j..64+8j+7, so RoPE needs no shuffle; the dot product
// is reduced over eight lanes; the online softmax runs once per step for
// four positions; P.V accumulates the lane's 16 elements of the rotated
// value.  RoPE angles: the lane's eight frequencies at its position, reduced
// in fp64 at the warp's first step and every 64 steps, advanced by 4*theta_f
// per step in between.
constexpr int PRQ_POS = 4;              // positions per warp step
constexpr int PRQ_REANCHOR = 64;        // steps between fp64 angle reductions
// Row stride (floats) of a position's channel-order key in shared memory:
// the four positions of a step scatter to the same channels, and the pad
// of 8 puts them in four different bank octets.
constexpr int PRQ_ROW = D + 8;

__device__ __forceinline__ void prq_angles(const PreRopeArgs &a, int t, int j, float (&cs)[8],
                                           float (&sn)[8]) {
#pragma unroll
    for (int m = 0; m < 8; m++) {
        const double u = (double)t * a.phi[8 * j + m];
        sincospif((float)(2.0 * (u - floor(u))), &sn[m], &cs[m]);
    }
}

// The codes and {s, z} of one position that a lane reads: its logical K
// word, its two V pieces and the four groups' K and V metadata.
struct PrqLoad {
    uint32_t kw, vw, km[4], vm[4];
};

__device__ __forceinline__ void prq_load(const PreRopeArgs &a, int b, int h, int t, int j,
                                         PrqLoad &d) {
    const long long bi = cache_block_index(a.table, a.num_blocks, a.nblk, a.Hkv, b, h, t / BLK_TOK);
    if (bi < 0 && j == 0) set_status(a.status, KVQ_DEV_BAD_TABLE);
    const uint8_t *bp = a.blocks + (size_t)(bi < 0 ? 0 : bi) * BLK_BYTES;
    const int tau = t % BLK_TOK, r = tau & 7, th = tau >> 3, q2 = tau >> 1;
    d.kw = *reinterpret_cast<const uint32_t *>(bp + 16 * (4 * r + (j & 3)) + 4 * (2 * th + (j >> 2)));
    const int vo = 512 + 16 * (q2 & 3) + 4 * (2 * (q2 >> 2) + (j >> 2)) + 2 * (tau & 1);
    const uint32_t v0 = *reinterpret_cast<const uint16_t *>(bp + vo + 64 * ((2 * j) & 7));
    const uint32_t v1 = *reinterpret_cast<const uint16_t *>(bp + vo + 64 * ((2 * j + 1) & 7));
    d.vw = v0 | (v1 << 16);
#pragma unroll
    for (int g = 0; g < 4; g++) {
        d.km[g] = *reinterpret_cast<const uint32_t *>(bp + 1024 + 8 * (4 * r + g) + 4 * th);
        d.vm[g] = *reinterpret_cast<const uint32_t *>(bp + 1280 + 8 * (4 * r + g) + 4 * th);
    }
}

__global__ void __launch_bounds__(PR_THREADS) prerope_split_q_kernel(PreRopeArgs a) {
    // Tables laid out so that the eight lanes of a position (j = 0..7) read
    // consecutive words: no bank conflicts.
    __shared__ __align__(16) float kb_s[PR_WARPS][PRQ_POS][PRQ_ROW];   // keys, channel order
    __shared__ __align__(16) float2 step_s[8][8];     // [m][j]: cos, sin of 4 theta_(8j+m)
    __shared__ __align__(16) float4 q_s[4][8];        // [quarter][j]: the query, exp2 domain
    __shared__ __align__(16) uint4 off_s[2][8];       // [half][j]: lane j's scatter offsets
    __shared__ float m_s[PR_WARPS], l_s[PR_WARPS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pp = lane >> 3, j = lane & 7;                     // position slot, lane in position
    const int split = blockIdx.x;
    const int b = blockIdx.y / a.Hkv, h = blockIdx.y % a.Hkv;
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x < D) {
        // channel c: quarter (c >= 64) * 2 + (c % 8) / 4 of lane j = (c % 64) / 8
        const int c = threadIdx.x, jj = (c & 63) >> 3, qu = 2 * (c >> 6) + ((c & 7) >> 2);
        reinterpret_cast<float *>(&q_s[qu][jj])[c & 3] =
            __half2float(__ushort_as_half(a.Q[((size_t)b * a.Hq + h) * D + c])) *
            (PR_LOG2E * 0.08838834764831845f);
        if (c < D / 2) {
            float sn4, cs4;
            const double u = 4.0 * a.phi[c];
            sincospif((float)(2.0 * (u - floor(u))), &sn4, &cs4);
            step_s[c & 7][c >> 3] = make_float2(cs4, sn4);
        }
    } else if (threadIdx.x < D + 64) {
        // word w = 2g + k/2 of lane jj (k = 0, 2): perm[32g + 4jj + k] |
        // perm[32g + 4jj + k + 1] << 16, where two elements of a position's
        // un-rotated key go in its channel-order row
        const int i = threadIdx.x - D, jj = i >> 3, w = i & 7, g = w >> 1, k = 2 * (w & 1);
        const int32_t *pm = a.perm + (size_t)h * D + 32 * g + 4 * jj + k;
        reinterpret_cast<uint32_t *>(&off_s[w >> 2][jj])[w & 3] =
            (uint32_t)(pm[0] & (D - 1)) | ((uint32_t)(pm[1] & (D - 1)) << 16);
    }
    const int L = a.seq_lens[b];
    const bool lok = L >= 1 && L <= a.capacity;
    const int nb = lok ? (L + BLK_TOK - 1) / BLK_TOK : 0;
    const int blk0 = split * a.bps, blk1 = min(nb, blk0 + a.bps);
    __syncthreads();                                   // q_s, step_s, off_s
    float *krow = &kb_s[warp][pp][0];

    // the CTA's tokens in PR_WARPS contiguous, equal runs, one per warp
    const int t_beg = min(L, max(a.S, blk0 * BLK_TOK)), t_end = max(t_beg, min(L, blk1 * BLK_TOK));
    const int per = (t_end - t_beg + PR_WARPS - 1) / PR_WARPS;
    const int w0 = min(t_end, t_beg + warp * per), w1 = min(t_end, w0 + per);

    float m_run = PR_M0, l_run = 0.f, o[16], zacc[4];
#pragma unroll
    for (int i = 0; i < 16; i++) o[i] = 0.f;
#pragma unroll
    for (int g = 0; g < 4; g++) zacc[g] = 0.f;
    float cs[8], sn[8];
    PrqLoad cur, nxt;
    if (w0 < w1) prq_load(a, b, h, min(w0 + pp, w1 - 1), j, cur);
    int step = 0;
    for (int tb = w0; tb < w1; tb += PRQ_POS, ++step) {
        const int t = tb + pp;
        const bool valid = t < w1;
        // the next step's loads in flight during this one (positions past
        // the run reload the run's last position)
        if (tb + PRQ_POS < w1) prq_load(a, b, h, min(tb + PRQ_POS + pp, w1 - 1), j, nxt);
        // the block two ahead into L2 (its 1536 bytes are 12 lines)
        if ((tb & (BLK_TOK - 1)) < PRQ_POS && pp == 0 && tb + 2 * BLK_TOK < w1) {
            const long long bn = cache_block_index(a.table, a.num_blocks, a.nblk, a.Hkv, b, h,
                                                   tb / BLK_TOK + 2);
            if (bn >= 0) {
                const uint8_t *pf = a.blocks + (size_t)bn * BLK_BYTES + 128 * j;
                asm volatile("prefetch.global.L2 [%0];" ::"l"(pf));
                if (j < 4) asm volatile("prefetch.global.L2 [%0];" ::"l"(pf + 1024));
            }
        }
        if (step % PRQ_REANCHOR == 0) {
            prq_angles(a, valid ? t : tb, j, cs, sn);
        } else {
#pragma unroll
            for (int m = 0; m < 8; m++) {
                const float2 st = step_s[m][j];
                const float c2 = cs[m] * st.x - sn[m] * st.y;
                sn[m] = fmaf(sn[m], st.x, cs[m] * st.y);
                cs[m] = c2;
            }
        }
        // ---- key: dequantise (1/sqrt(128) folded into s and z), FWHT, scatter
        float v[16];
#pragma unroll
        for (int g = 0; g < 4; g++) {
            const float2 sz = unpack_half2(cur.km[g]);
            const float s = sz.x * 0.08838834764831845f, z = sz.y * 0.08838834764831845f;
            float c[4];
            unpack4(cur.kw, g, c);
#pragma unroll
            for (int k = 0; k < 4; k++) v[4 * g + k] = fmaf(c[k], s, z);
        }
        // in-lane stages: v[4g + k] holds element 32g + 4j + k, so the
        // strides 1, 2 are index bits 0, 1 (k) and 4, 8 are bits 5, 6 (g)
#pragma unroll
        for (int st = 1; st < 16; st <<= 1)
#pragma unroll
            for (int i = 0; i < 16; i++)
                if ((i & st) == 0) {
                    const float x0 = v[i], x1 = v[i + st];
                    v[i] = x0 + x1;
                    v[i + st] = x0 - x1;
                }
        // cross-lane stages: index bits 2, 3, 4 (j)
#pragma unroll
        for (int mk = 1; mk < 8; mk <<= 1) {
            const float sgn = (j & mk) ? -1.f : 1.f;
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const float o2 = __shfl_xor_sync(0xffffffffu, v[i], mk);
                v[i] = fmaf(sgn, v[i], o2);
            }
        }
        // k_pre[perm[e]] = y[e]
        {
            const uint4 oa = off_s[0][j];
            const uint4 ob4 = off_s[1][j];
            const uint32_t off2[8] = {oa.x, oa.y, oa.z, oa.w, ob4.x, ob4.y, ob4.z, ob4.w};
#pragma unroll
            for (int w = 0; w < 8; w++) {
                krow[off2[w] & 0xffffu] = v[2 * w];
                krow[off2[w] >> 16] = v[2 * w + 1];
            }
        }
        __syncwarp();
        float x[8], xp[8];
        {
            const float4 a0 = *reinterpret_cast<const float4 *>(krow + 8 * j);
            const float4 a1 = *reinterpret_cast<const float4 *>(krow + 8 * j + 4);
            const float4 b0 = *reinterpret_cast<const float4 *>(krow + 64 + 8 * j);
            const float4 b1 = *reinterpret_cast<const float4 *>(krow + 64 + 8 * j + 4);
            x[0] = a0.x; x[1] = a0.y; x[2] = a0.z; x[3] = a0.w;
            x[4] = a1.x; x[5] = a1.y; x[6] = a1.z; x[7] = a1.w;
            xp[0] = b0.x; xp[1] = b0.y; xp[2] = b0.z; xp[3] = b0.w;
            xp[4] = b1.x; xp[5] = b1.y; xp[6] = b1.z; xp[7] = b1.w;
        }
        __syncwarp();
        // RoPE at position t (channel c < 64 with its partner c + 64) and the
        // dot with the query over this lane's 16 channels
        float d = 0.f;
        {
            const float4 qa0 = q_s[0][j], qa1 = q_s[1][j], qb0 = q_s[2][j], qb1 = q_s[3][j];
            const float qa[8] = {qa0.x, qa0.y, qa0.z, qa0.w, qa1.x, qa1.y, qa1.z, qa1.w};
            const float qb[8] = {qb0.x, qb0.y, qb0.z, qb0.w, qb1.x, qb1.y, qb1.z, qb1.w};
#pragma unroll
            for (int m = 0; m < 8; m++) {
                const float xr = fmaf(-xp[m], sn[m], x[m] * cs[m]);
                const float xpr = fmaf(x[m], sn[m], xp[m] * cs[m]);
                d = fmaf(qa[m], xr, d);
                d = fmaf(qb[m], xpr, d);
            }
        }
        d += __shfl_xor_sync(0xffffffffu, d, 1);
        d += __shfl_xor_sync(0xffffffffu, d, 2);
        d += __shfl_xor_sync(0xffffffffu, d, 4);
        // an identified sink's slot (NaN scale) scores NaN: fmax with -inf
        // makes it -inf, weight 0 (m_run starts at PR_M0, finite)
        d = valid ? fmaxf(d, PR_NEG_INF) : PR_NEG_INF;
        // ---- online softmax over the step's four positions
        float mx = fmaxf(d, __shfl_xor_sync(0xffffffffu, d, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        if (mx > m_run) {                              // uniform over the warp
            const float al = fast_exp2(m_run - mx);
            l_run *= al;
#pragma unroll
            for (int i = 0; i < 16; i++) o[i] *= al;
#pragma unroll
            for (int g = 0; g < 4; g++) zacc[g] *= al;
            m_run = mx;
        }
        const float p = fast_exp2(d - m_run);
        l_run += p;
        // ---- P.V on the rotated value: o += (p s) c, zacc += p z per group
#pragma unroll
        for (int g = 0; g < 4; g++) {
            const float2 sz = unpack_half2(cur.vm[g]);
            float c[4];
            unpack4(cur.vw, g, c);
            const float ps = p * sz.x;
#pragma unroll
            for (int k = 0; k < 4; k++) o[4 * g + k] = fmaf(ps, c[k], o[4 * g + k]);
            zacc[g] = fmaf(p, sz.y, zacc[g]);
        }
        cur = nxt;
    }
    // the four position slots hold partial sums over different positions
#pragma unroll
    for (int i = 0; i < 16; i++) {
        o[i] += __shfl_xor_sync(0xffffffffu, o[i], 8);
        o[i] += __shfl_xor_sync(0xffffffffu, o[i], 16);
    }
#pragma unroll
    for (int g = 0; g < 4; g++) {
        zacc[g] += __shfl_xor_sync(0xffffffffu, zacc[g], 8);
        zacc[g] += __shfl_xor_sync(0xffffffffu, zacc[g], 16);
    }
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);

    // combine the warps through kb_s, reused as [PR_WARPS][128]
    __syncthreads();
    float *ob = &kb_s[0][0][0];
    static_assert(PR_WARPS * D <= PR_WARPS * PRQ_POS * PRQ_ROW, "combine area");
    if (pp == 0) {
#pragma unroll
        for (int g = 0; g < 4; g++)
#pragma unroll
            for (int k = 0; k < 4; k++) ob[warp * D + 32 * g + 4 * j + k] = o[4 * g + k] + zacc[g];
        if (j == 0) {
            m_s[warp] = m_run;
            l_s[warp] = l_run;
        }
    }
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += PR_THREADS) {
        float mx = PR_NEG_INF;
#pragma unroll
        for (int w = 0; w < PR_WARPS; w++) mx = fmaxf(mx, m_s[w]);
        float lt = 0.f, ot = 0.f;
#pragma unroll
        for (int w = 0; w < PR_WARPS; w++) {
            const float f = exp2f(m_s[w] - mx);        // PR_M0 runs (no tokens): l = 0, o = 0
            lt = fmaf(f, l_s[w], lt);
            ot = fmaf(f, ob[w * D + c], ot);
        }
        float *pp2 = a.part + (((size_t)b * a.Hq + h) * a.nsplit + split) * PR_PART;
        pp2[4 + c] = ot;
        if (c == 0) {
            pp2[0] = mx;
            pp2[1] = lt;
        }
    }
}

// Merge of the splits and the inverse value rotation, one CTA of 128
// threads per (b, query head).
__global__ void __launch_bounds__(D) prerope_merge_kernel(PreRopeArgs a) {
    __shared__ __align__(16) float os[D];
    __shared__ float red4[D / 32];
    const int hq = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
    const int h = hq / (a.Hq / a.Hkv);
    pdl_wait();
    pdl_trigger();
    const int L = a.seq_lens[b];
    uint16_t *out = a.out + ((size_t)b * a.Hq + hq) * D;
    if (L < 1 || L > a.capacity) {
        out[t] = 0;
        if (t == 0) set_status(a.status, KVQ_DEV_BAD_LEN);
        return;
    }
    // ---- the fp16 sinks this query sees, scored on CUDA cores: the stored
    // pre-RoPE key turned by RoPE at the sink's position (thread t = channel
    // t, its pair partner t ^ 64), dotted with q; softmax partial over them
    int ns = 0;
    if (a.Srows > 0) {
        if (!a.sink_pos) {
            ns = min(a.S, L);
        } else {
            const int n = min(max(a.sink_count[b], 0), a.Srows);
            for (int r = 0; r < n; r++) ns += a.sink_pos[(size_t)b * a.Srows + r] < L ? 1 : 0;
        }
    }
    float sm = PR_NEG_INF, sl = 0.f, so = 0.f;
    if (ns > 0) {
        const size_t uh = (size_t)b * a.Hkv + h;
        const uint16_t *ks = a.k_sink + uh * a.Srows * D;
        const uint16_t *vs = a.v_sink + uh * a.Srows * D;
        const float qv = __half2float(__ushort_as_half(a.Q[((size_t)b * a.Hq + hq) * D + t])) *
                         (PR_LOG2E * 0.08838834764831845f);
        const double ph = a.phi[t & (D / 2 - 1)];
        const float sgn = t < D / 2 ? -1.f : 1.f;
        const int lane = t & 31, warp = t >> 5;
        for (int r = 0; r < ns; r++) {
            const int pos = a.sink_pos ? a.sink_pos[(size_t)b * a.Srows + r] : r;
            const double u = (double)pos * ph;
            float sn, cs;
            sincospif((float)(2.0 * (u - floor(u))), &sn, &cs);
            const float x = __half2float(__ushort_as_half(ks[(size_t)r * D + t]));
            const float xp = __half2float(__ushort_as_half(ks[(size_t)r * D + (t ^ (D / 2))]));
            float d = qv * fmaf(sgn * xp, sn, x * cs);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
            if (lane == 0) red4[warp] = d;
            __syncthreads();
            const float sc = red4[0] + red4[1] + red4[2] + red4[3];
            __syncthreads();
            const float mnew = fmaxf(sm, sc);
            const float al = sm == PR_NEG_INF ? 0.f : exp2f(sm - mnew);
            const float p = exp2f(sc - mnew);
            sl = fmaf(sl, al, p);
            so = fmaf(so, al, p * __half2float(__ushort_as_half(vs[(size_t)r * D + t])));
            sm = mnew;
        }
    }
    const float *pp = a.part + ((size_t)b * a.Hq + hq) * a.nsplit * PR_PART;
    float mx = sm;
    for (int s = 0; s < a.nsplit; s++) mx = fmaxf(mx, pp[(size_t)s * PR_PART]);
    float lt = 0.f, ot = 0.f;
    if (sm != PR_NEG_INF) {
        const float f = exp2f(sm - mx);
        lt = f * sl;
        ot = f * so;
    }
    for (int s = 0; s < a.nsplit; s++) {
        const float ms = pp[(size_t)s * PR_PART];
        if (ms == PR_NEG_INF) continue;                     // a split without tokens
        const float f = exp2f(ms - mx);
        lt = fmaf(f, pp[(size_t)s * PR_PART + 1], lt);
        ot = fmaf(f, pp[(size_t)s * PR_PART + 4 + t], ot);
    }
    os[t] = lt > 0.f ? ot / lt : 0.f;
    __syncthreads();
    if (t < 32) {
        float v[4] = {os[4 * t], os[4 * t + 1], os[4 * t + 2], os[4 * t + 3]};
        fwht128_warp(v);
        const int4 pi = *reinterpret_cast<const int4 *>(a.perm + ((size_t)a.Hkv + h) * D + 4 * t);
        out[pi.x & (D - 1)] = __half_as_ushort(__float2half_rn(v[0] * 0.08838834764831845f));
        out[pi.y & (D - 1)] = __half_as_ushort(__float2half_rn(v[1] * 0.08838834764831845f));
        out[pi.z & (D - 1)] = __half_as_ushort(__float2half_rn(v[2] * 0.08838834764831845f));
        out[pi.w & (D - 1)] = __half_as_ushort(__float2half_rn(v[3] * 0.08838834764831845f));
    }
}

size_t prerope_ws_bytes(int B, int Hq, int Hkv, int gh, int max_ctx, int sms) {
    const int ns = pr_nsplit(B, Hkv / gh, max_ctx, sms);
    return sizeof(float) * (size_t)B * Hq * ns * PR_PART;
}

template <int GH, int G>
static cudaError_t launch_split_pr(const PreRopeArgs &a, cudaStream_t st) {
    return launch_pdl(prerope_split_kernel<GH, G>, dim3(a.nsplit, a.B * (a.Hkv / GH)),
                      dim3(PR_THREADS), 0, st, a);
}

cudaError_t launch_decode_prerope(const uint16_t *Q, int Hq, const kvq_cache_desc &cd, int gh,
                                  const int32_t *perm, float rope_base, const int32_t *seq_lens,
                                  int max_ctx, int sms, void *ws, uint16_t *out, cudaStream_t st) {
    PreRopeArgs a;
    a.Q = Q;
    a.blocks = static_cast<const uint8_t *>(cd.blocks);
    a.table = cd.block_table;
    a.num_blocks = cd.num_blocks;
    a.perm = perm;
    a.seq_lens = seq_lens;
    a.status = cd.status;
    a.part = static_cast<float *>(ws);
    a.out = out;
    a.k_sink = cd.k_sink;
    a.v_sink = cd.v_sink;
    a.sink_pos = cd.sink_pos;
    a.sink_count = cd.sink_count;
    a.Srows = cd.sink_fp16;
    a.S = cd.sink_pos ? 0 : cd.sink_fp16;
    a.B = cd.B;
    a.Hq = Hq;
    a.Hkv = cd.Hkv;
    a.capacity = cd.capacity;
    a.nblk = cd.capacity / BLK_TOK;
    a.nsplit = pr_nsplit(cd.B, cd.Hkv / gh, max_ctx, sms);
    const int nb = (max_ctx + BLK_TOK - 1) / BLK_TOK;
    a.bps = (nb + a.nsplit - 1) / a.nsplit;
    // theta_f / (2 pi) in fp64: the kernel reduces t * theta_f modulo 2 pi
    for (int f = 0; f < D / 2; f++)
        a.phi[f] = pow((double)rope_base, -2.0 * f / D) / (2.0 * 3.14159265358979323846);
    const int G = Hq / cd.Hkv;
    cudaError_t e;
    switch (gh * 16 + G) {
        case 1 * 16 + 1:
            e = launch_pdl(prerope_split_q_kernel, dim3(a.nsplit, a.B * a.Hkv), dim3(PR_THREADS), 0,
                           st, a);
            break;
        case 1 * 16 + 2: e = launch_split_pr<1, 2>(a, st); break;
        case 1 * 16 + 4: e = launch_split_pr<1, 4>(a, st); break;
        case 1 * 16 + 8: e = launch_split_pr<1, 8>(a, st); break;
        case 2 * 16 + 1: e = launch_split_pr<2, 1>(a, st); break;
        case 2 * 16 + 2: e = launch_split_pr<2, 2>(a, st); break;
        case 2 * 16 + 4: e = launch_split_pr<2, 4>(a, st); break;
        case 4 * 16 + 1: e = launch_split_pr<4, 1>(a, st); break;
        case 4 * 16 + 2: e = launch_split_pr<4, 2>(a, st); break;
        case 8 * 16 + 1: e = launch_split_pr<8, 1>(a, st); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    return launch_pdl(prerope_merge_kernel, dim3(Hq, cd.B), dim3(D), 0, st, a);
}

}  // namespace kvq
