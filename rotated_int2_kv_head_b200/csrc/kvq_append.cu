// Rotate -> quantize -> append kernels (CUDA cores).
//
// Method: each KV head owns an orthogonal rotation applied to keys and values
// before INT2 quantization ("Output-Aware Rotation for INT2 KV-Cache
// Quantization", section "Key Details"), either a dense 128x128 matrix or a
// channel reordering followed by a fast Walsh-Hadamard transform ("RotateKV",
// abstract item (i); "KVLinC", abstract).  The first positions of every
// sequence are attention sinks kept in fp16 ("RotateKV", item (iii)).
//
// Kernels here:
//   append_dense_kernel  dense rotation on CUDA cores; R is held in registers
//                        and reused across the tokens of a CTA (small and
//                        medium T; large T goes to the tensor-core kernel).
//   append_fwht_kernel   one warp per row: permutation gather, 128-point FWHT
//                        in registers and shuffles, quantize, pack.
//   The last CTA of an append to finish adds T to every valid seq_lens[b]
//   (a completion counter in the cache's second status word tells it that it
//   is last), so no separate kernel is needed.
//   debug kernels        the same rotation / quantizer code with fp32 outputs.
#include "kvq_internal.cuh"

namespace kvq {

// Epilogue shared by the append kernels: row (b, t, h, kind) with rotated
// values v (lane layout of quantize_row_warp).  A sink stores v in fp16, or,
// when raw is given, the lane's 4 halves of the row as it came in (the
// pre-RoPE mode keeps sink keys unrotated).
__device__ __forceinline__ void cache_epilogue(const CacheDst &c, int b, int t, int h, int kind,
                                               int L0, const float v[4],
                                               const uint16_t *raw = nullptr) {
    const int lane = threadIdx.x & 31;
    const int p = L0 + t;
    const long long bi = cache_block_index(c.table, c.num_blocks, c.nblk, c.Hkv, b, h, p / BLK_TOK);
    if (bi < 0 && lane == 0) set_status(c.status, KVQ_DEV_BAD_TABLE);
    uint8_t *block = c.blocks + (size_t)(bi < 0 ? 0 : bi) * BLK_BYTES;
    const int tau = p % BLK_TOK;
    const int row = sink_row(c, b, p);                 // uniform over the warp
    if (row >= 0) {
        uint16_t *sink = (kind == 0 ? c.k_sink : c.v_sink) +
                         (((size_t)b * c.Hkv + h) * c.S + (size_t)row) * D + 4 * lane;
        uint2 pk;
        if (raw) {          // the row as given (pre-RoPE keys), the lane's 4 halves
            pk = *reinterpret_cast<const uint2 *>(raw);
        } else {
            pk.x = pack_half2(v[0], v[1]);
            pk.y = pack_half2(v[2], v[3]);
        }
        *reinterpret_cast<uint2 *>(sink) = pk;
        if (bi >= 0) {
            // zero codes and meta; an identified sink's K meta carries the marker
            QuantWord q;
            q.word = 0;
            q.s = (c.sink_pos && kind == 0) ? (uint16_t)SINK_KMETA_MARK : (uint16_t)0;
            q.z = 0;
            store_token_warp(block, tau, kind, q);
        }
    } else {
        const QuantWord q = quantize_row_warp(v);      // warp-collective: every lane runs it
        if (bi >= 0) store_token_warp(block, tau, kind, q);
    }
}

// ---- dense rotation on CUDA cores ---------------------------------------------------------
// 256 threads.  Warp w owns rows 16w..16w+15 of R, lane l columns 4l..4l+3:
// a 16x4 register tile, reused for every row of the CTA.  Rows go in
// batches of 8: every warp forms its partial dot products for all 8, the
// partials are summed in a fixed order through shared memory, and warp k
// finishes row k of the batch (quantize + store, or fp32 store).  In cache
// mode a CTA takes one (head, K|V) and the rows (b, t) of `bpc` consecutive
// sequences b times a chunk of `tchunk` tokens t: appends of a few tokens
// to many sequences (a decode step) share one fetch of R between
// sequences.
constexpr int DENSE_THREADS = 256;
constexpr int DENSE_BATCH = 8;

struct DenseRows {
    // cache mode: grid (tchunks, Hkv, 2*ceil(B/bpc)); debug mode: grid (chunks, 1, 1)
    const uint16_t *X0, *X1;   // K, V (cache) or X (debug)
    const float *R0, *R1;      // R_k, R_v [Hkv][128][128] (cache) or R (debug)
    float *out_f32;            // debug output or nullptr
    int n_rows;                // debug: N
    int tchunk;                // tokens (rows) per CTA and sequence
    int bpc;                   // cache mode: sequences per CTA (1..DENSE_BATCH)
};

template <bool TO_CACHE>
__global__ void __launch_bounds__(DENSE_THREADS)
    append_dense_kernel(DenseRows a, CacheDst c) {
    __shared__ __align__(16) uint16_t xs[DENSE_BATCH][D];
    __shared__ __align__(16) float red[DENSE_BATCH][8][D];
    __shared__ int L0s[DENSE_BATCH];            // cache mode: start length per sequence
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int b0 = 0, nseq = 1, h = 0, kind = 0, row0;
    const uint16_t *X;
    const float *R;
    if (TO_CACHE) {
        h = blockIdx.y;
        kind = blockIdx.z & 1;
        b0 = (int)(blockIdx.z >> 1) * a.bpc;
        nseq = min(a.bpc, c.B - b0);
        X = (kind == 0 ? a.X0 : a.X1);
        R = (kind == 0 ? a.R0 : a.R1) + (size_t)h * D * D;
    } else {
        X = a.X0;
        R = a.R0;
    }
    // R (a rotation input, never written by the work this kernel waits on) is
    // fetched before the dependency wait, overlapping the preceding kernel
    float Rr[16][4];
#pragma unroll
    for (int ii = 0; ii < 16; ii++) {
        const float4 r4 = *reinterpret_cast<const float4 *>(R + (16 * warp + ii) * D + 4 * lane);
        Rr[ii][0] = r4.x;
        Rr[ii][1] = r4.y;
        Rr[ii][2] = r4.z;
        Rr[ii][3] = r4.w;
    }
    pdl_wait();
    pdl_trigger();
    row0 = blockIdx.x * a.tchunk;
    const int avail = min(a.tchunk, (TO_CACHE ? c.T : a.n_rows) - row0);   // >= 1 by the grid
    // row i of the CTA: sequence b0 + i / avail, token row0 + i % avail
    const int nrows = nseq * avail;
    // thread t stages 16 B of row (base + t/16) of a batch: 8 rows x 256 B
    const int rr = threadIdx.x >> 4, piece = threadIdx.x & 15;
    auto piece_ptr = [&](int i) -> const uint4 * {
        const int b = b0 + i / avail, row = row0 + i % avail;
        const uint16_t *src = TO_CACHE ? X + (((size_t)b * c.T + row) * c.Hkv + h) * D
                                       : X + (size_t)row * D;
        return reinterpret_cast<const uint4 *>(src + piece * 8);
    };
    // the first batch's input is loaded before seq_lens is examined: the two
    // loads are independent and overlap
    uint4 first = make_uint4(0u, 0u, 0u, 0u);
    if (rr < min(DENSE_BATCH, nrows)) first = *piece_ptr(rr);
    unsigned claim = 0u;
    if (TO_CACHE) {
        // a skipped sequence (no room, negative length) stores no rows; the
        // first column of CTAs reports it
        if (threadIdx.x < nseq)
            L0s[threadIdx.x] = start_len_thread(c, b0 + threadIdx.x,
                                                blockIdx.x == 0 && blockIdx.y == 0 && kind == 0);
        claim = append_claim(c);                             // seq_lens is not read again
    }

    for (int base = 0; base < nrows; base += DENSE_BATCH) {
        const int nb = min(DENSE_BATCH, nrows - base);
        if (rr < nb)
            *reinterpret_cast<uint4 *>(&xs[rr][piece * 8]) =
                base == 0 ? first : *piece_ptr(base + rr);
        __syncthreads();
        for (int k = 0; k < nb; k++) {
            const uint4 u0 = *reinterpret_cast<const uint4 *>(&xs[k][16 * warp]);
            const uint4 u1 = *reinterpret_cast<const uint4 *>(&xs[k][16 * warp + 8]);
            const uint32_t w8[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ii = 0; ii < 8; ii++) {
                const float2 x2 = unpack_half2(w8[ii]);
#pragma unroll
                for (int cc = 0; cc < 4; cc++) {
                    acc[cc] = fmaf(x2.x, Rr[2 * ii][cc], acc[cc]);
                    acc[cc] = fmaf(x2.y, Rr[2 * ii + 1][cc], acc[cc]);
                }
            }
            *reinterpret_cast<float4 *>(&red[k][warp][4 * lane]) =
                make_float4(acc[0], acc[1], acc[2], acc[3]);
        }
        __syncthreads();
        if (warp < nb) {
            float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int w2 = 0; w2 < 8; w2++) {
                const float4 p4 = *reinterpret_cast<const float4 *>(&red[warp][w2][4 * lane]);
                v[0] += p4.x;
                v[1] += p4.y;
                v[2] += p4.z;
                v[3] += p4.w;
            }
            const int i = base + warp;
            if (TO_CACHE) {
                const int L0 = L0s[i / avail];               // uniform over the warp
                if (L0 >= 0) cache_epilogue(c, b0 + i / avail, row0 + i % avail, h, kind, L0, v);
            } else {
                const int row = row0 + i;
                *reinterpret_cast<float4 *>(a.out_f32 + (size_t)row * D + 4 * lane) =
                    make_float4(v[0], v[1], v[2], v[3]);
            }
        }
        __syncthreads();
    }
    if (TO_CACHE) append_finish(c, claim);
}

// ---- permutation + FWHT ---------------------------------------------------------------------
// One warp per row: y[i] = x[perm[i]], y <- FWHT(y) / sqrt(128).
constexpr int FWHT_THREADS = 256;
constexpr int FWHT_ROWS = FWHT_THREADS / 4;   // rows per CTA: four threads per row
// Staged rows are 272 bytes apart: the 8 rows of a warp that gather the same
// permuted index then fall in 8 different shared-memory banks (at 256 bytes
// they would all share one).
constexpr int XS_STRIDE = D + 8;

struct FwhtRows {
    const uint16_t *X0, *X1;   // K, V (cache) or X (debug)
    const int32_t *perm;       // [2][Hkv][128] (cache) or [128] (debug)
    float *out_f32;
    long long n_rows;          // cache: B*T*Hkv*2 ; debug: N
};

// Thread q (0..3) of a row staged in shared memory: its 32 elements of
// FWHT(x[perm]) / sqrt(128), elements 32q .. 32q+31 (quantization group q).
// Five butterfly stages run in registers, the two over index bits 5 and 6
// across the row's four consecutive lanes.  Every lane of the warp calls it
// (shuffles); a row that is not active computes zeros.
__device__ __forceinline__ void fwht_row_quarter(const uint16_t *xrow, const int32_t *perm,
                                                 bool active, int q, float (&v)[32]) {
#pragma unroll
    for (int i = 0; i < 8; i++) {
        int4 pi = make_int4(0, 0, 0, 0);
        if (active) pi = *reinterpret_cast<const int4 *>(perm + 32 * q + 4 * i);
        v[4 * i] = active ? __half2float(__ushort_as_half(xrow[pi.x & (D - 1)])) : 0.f;
        v[4 * i + 1] = active ? __half2float(__ushort_as_half(xrow[pi.y & (D - 1)])) : 0.f;
        v[4 * i + 2] = active ? __half2float(__ushort_as_half(xrow[pi.z & (D - 1)])) : 0.f;
        v[4 * i + 3] = active ? __half2float(__ushort_as_half(xrow[pi.w & (D - 1)])) : 0.f;
    }
#pragma unroll
    for (int st = 1; st < 32; st <<= 1)
#pragma unroll
        for (int e = 0; e < 32; e++)
            if ((e & st) == 0) {
                const float x0 = v[e], x1 = v[e + st];
                v[e] = x0 + x1;
                v[e + st] = x0 - x1;
            }
#pragma unroll
    for (int m = 1; m < 4; m <<= 1) {
        const float sgn = (q & m) ? -1.f : 1.f;
#pragma unroll
        for (int e = 0; e < 32; e++) {
            const float o = __shfl_xor_sync(0xffffffffu, v[e], m);
            v[e] = fmaf(sgn, v[e], o);
        }
    }
    scale_group(v, 0.08838834764831845f);
}

// Four threads per row.  Thread q (0..3) owns elements 32q..32q+31 of the
// rotated row, which is exactly quantization group q: the FWHT's five
// stages over index bits 0..4 run in its registers, the two over bits 5 and
// 6 across the row's four threads (consecutive lanes: shuffles xor 1 and 2,
// each butterfly one fma with a per-thread sign), and then the thread
// quantizes its group alone (quantize_group_thread); the row's code words
// are OR-ed together over its four threads.  The row is gathered through
// the permutation from shared memory.  Cache: CTA (bt, y) takes token
// bt = b*T + t and the (head, kind) pairs 64y .. 64y+63 (kind fastest);
// debug: rows 64x .. 64x+63.
template <bool TO_CACHE>
__global__ void __launch_bounds__(FWHT_THREADS) append_fwht_kernel(FwhtRows a, CacheDst c) {
    __shared__ __align__(16) uint16_t xs[FWHT_ROWS][XS_STRIDE];
    const int r = threadIdx.x >> 2, q = threadIdx.x & 3;
    pdl_wait();
    pdl_trigger();
    const long long row = TO_CACHE ? 0 : (long long)blockIdx.x * FWHT_ROWS + r;
    const int hk = TO_CACHE ? (int)blockIdx.y * FWHT_ROWS + r : 0;
    bool active = TO_CACHE ? hk < 2 * c.Hkv : row < a.n_rows;
    int b = 0, t = 0, h = 0, kind = 0, L0 = 0;
    const uint16_t *src = nullptr;
    const int32_t *perm = nullptr;
    if (active && TO_CACHE) {
        kind = hk & 1;
        h = hk >> 1;
        b = (int)(blockIdx.x / (unsigned)c.T);
        t = (int)(blockIdx.x - (unsigned)b * (unsigned)c.T);
        L0 = start_len_thread(c, b, q == 0 && t == 0 && h == 0 && kind == 0);
        if (L0 < 0) active = false;
        src = (kind == 0 ? a.X0 : a.X1) + (((size_t)b * c.T + t) * c.Hkv + h) * D;
        perm = a.perm + ((size_t)kind * c.Hkv + h) * D;
    } else if (active) {
        src = a.X0 + (size_t)row * D;
        perm = a.perm;
    }
    // stage the row (thread q copies 64 of its 256 bytes)
    if (active) {
        const uint4 *s4 = reinterpret_cast<const uint4 *>(src) + 4 * q;
        uint4 *d4 = reinterpret_cast<uint4 *>(&xs[r][0]) + 4 * q;
#pragma unroll
        for (int i = 0; i < 4; i++) d4[i] = s4[i];
    }
    __syncwarp();
    float v[32];
    fwht_row_quarter(xs[r], perm, active, q, v);

    if (!TO_CACHE) {
        if (active) {
            float *dst = a.out_f32 + (size_t)row * D + 32 * q;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4 *>(dst + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
        return;
    }
    uint32_t words[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    uint32_t meta = quantize_group_thread(v, q, words);
#pragma unroll
    for (int w = 0; w < 8; w++) {
        words[w] |= __shfl_xor_sync(0xffffffffu, words[w], 1);
        words[w] |= __shfl_xor_sync(0xffffffffu, words[w], 2);
    }
    if (active) {
        const int p = L0 + t;
        const long long bi = cache_block_index(c.table, c.num_blocks, c.nblk, c.Hkv, b, h, p / BLK_TOK);
        if (bi < 0 && q == 0) set_status(c.status, KVQ_DEV_BAD_TABLE);
        uint8_t *block = c.blocks + (size_t)(bi < 0 ? 0 : bi) * BLK_BYTES;
        const int tau = p % BLK_TOK;
        const int srow = sink_row(c, b, p);
        if (srow >= 0) {
            // a sink: the rotated row in fp16; its slot zero (identified: K marker)
            uint16_t *dst = (kind == 0 ? c.k_sink : c.v_sink) +
                            (((size_t)b * c.Hkv + h) * c.S + (size_t)srow) * D + 32 * q;
#pragma unroll
            for (int e = 0; e < 32; e += 8)
                *reinterpret_cast<uint4 *>(dst + e) =
                    make_uint4(pack_half2(v[e], v[e + 1]), pack_half2(v[e + 2], v[e + 3]),
                               pack_half2(v[e + 4], v[e + 5]), pack_half2(v[e + 6], v[e + 7]));
#pragma unroll
            for (int w = 0; w < 8; w++) words[w] = 0u;
            meta = (c.sink_pos && kind == 0) ? SINK_KMETA_MARK : 0u;
        }
        // thread q stores code words 2q and 2q+1 (selected without indexing
        // the array by a runtime value, which would put it in local memory)
        uint32_t wa = words[0], wb = words[1];
#pragma unroll
        for (int k = 1; k < 4; k++)
            if (q == k) {
                wa = words[2 * k];
                wb = words[2 * k + 1];
            }
        if (bi >= 0) {
            if (kind == 0) {
                *reinterpret_cast<uint32_t *>(block + off_kword(tau, 2 * q)) = wa;
                *reinterpret_cast<uint32_t *>(block + off_kword(tau, 2 * q + 1)) = wb;
                *reinterpret_cast<uint32_t *>(block + off_kmeta(tau, q)) = meta;
            } else {                                    // 16-bit pieces 4q .. 4q+3
                *reinterpret_cast<uint16_t *>(block + off_vpiece(tau, 4 * q)) = (uint16_t)wa;
                *reinterpret_cast<uint16_t *>(block + off_vpiece(tau, 4 * q + 1)) = (uint16_t)(wa >> 16);
                *reinterpret_cast<uint16_t *>(block + off_vpiece(tau, 4 * q + 2)) = (uint16_t)wb;
                *reinterpret_cast<uint16_t *>(block + off_vpiece(tau, 4 * q + 3)) = (uint16_t)(wb >> 16);
                *reinterpret_cast<uint32_t *>(block + off_vmeta(tau, q)) = meta;
            }
        }
    }
    append_done(c);
}

// Bulk FWHT appends (T >= FWHT_CHUNK_MIN_T): CTA (chunk, 2h + kind, b)
// takes FWHT_ROWS consecutive new tokens of one (sequence, head, kind), four
// threads per row as above.  A cache block the chunk covers whole (16
// tokens) is assembled in shared memory and written out as the kind's
// 512-byte code region and 256-byte metadata region in 16-byte stores; the
// tokens of a block the chunk covers only in part are stored one by one.
constexpr int FWHT_CHUNK_MIN_T = 16;
constexpr int FWHT_TILE_BLKS = FWHT_ROWS / BLK_TOK + 1;   // blocks a chunk can touch

__global__ void __launch_bounds__(FWHT_THREADS) append_fwht_chunk_kernel(FwhtRows a, CacheDst c) {
    __shared__ __align__(16) uint16_t xs[FWHT_ROWS][XS_STRIDE];
    __shared__ __align__(16) uint8_t tile[FWHT_TILE_BLKS][BLK_BYTES];
    const int r = threadIdx.x >> 2, q = threadIdx.x & 3;
    const int kind = blockIdx.y & 1, h = blockIdx.y >> 1, b = blockIdx.z;
    const int t0 = blockIdx.x * FWHT_ROWS;
    pdl_wait();
    pdl_trigger();
    const int L0 = start_len_thread(c, b, threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0);
    const int nrows = min(FWHT_ROWS, c.T - t0);
    const bool active = L0 >= 0 && r < nrows;                 // L0 is uniform over the CTA
    const int32_t *perm = a.perm + ((size_t)kind * c.Hkv + h) * D;
    if (active) {
        const uint16_t *src = (kind == 0 ? a.X0 : a.X1) + (((size_t)b * c.T + t0 + r) * c.Hkv + h) * D;
        const uint4 *s4 = reinterpret_cast<const uint4 *>(src) + 4 * q;
        uint4 *d4 = reinterpret_cast<uint4 *>(&xs[r][0]) + 4 * q;
#pragma unroll
        for (int i = 0; i < 4; i++) d4[i] = s4[i];
    }
    __syncwarp();
    float v[32];
    fwht_row_quarter(xs[r], perm, active, q, v);
    uint32_t words[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    uint32_t meta = quantize_group_thread(v, q, words);
#pragma unroll
    for (int w = 0; w < 8; w++) {
        words[w] |= __shfl_xor_sync(0xffffffffu, words[w], 1);
        words[w] |= __shfl_xor_sync(0xffffffffu, words[w], 2);
    }
    uint32_t wa = words[0], wb = words[1];                     // thread q's words 2q, 2q+1
#pragma unroll
    for (int k = 1; k < 4; k++)
        if (q == k) {
            wa = words[2 * k];
            wb = words[2 * k + 1];
        }
    const int P0 = L0 + t0, P1 = P0 + nrows;                  // positions of the chunk
    const int lb0 = P0 / BLK_TOK;
    if (active) {
        const int p = P0 + r, lb = p / BLK_TOK, tau = p % BLK_TOK;
        const int srow = sink_row(c, b, p);
        if (srow >= 0) {
            uint16_t *dst = (kind == 0 ? c.k_sink : c.v_sink) +
                            (((size_t)b * c.Hkv + h) * c.S + (size_t)srow) * D + 32 * q;
#pragma unroll
            for (int e = 0; e < 32; e += 8)
                *reinterpret_cast<uint4 *>(dst + e) =
                    make_uint4(pack_half2(v[e], v[e + 1]), pack_half2(v[e + 2], v[e + 3]),
                               pack_half2(v[e + 4], v[e + 5]), pack_half2(v[e + 6], v[e + 7]));
            wa = wb = 0u;
            meta = (c.sink_pos && kind == 0) ? SINK_KMETA_MARK : 0u;
        }
        const bool whole = lb * BLK_TOK >= P0 && (lb + 1) * BLK_TOK <= P1;
        uint8_t *block;
        if (whole) {
            block = tile[lb - lb0];
        } else {
            const long long bi = cache_block_index(c.table, c.num_blocks, c.nblk, c.Hkv, b, h, lb);
            if (bi < 0 && q == 0) set_status(c.status, KVQ_DEV_BAD_TABLE);
            block = bi < 0 ? nullptr : c.blocks + (size_t)bi * BLK_BYTES;
        }
        if (block) {
            if (kind == 0) {
                *reinterpret_cast<uint32_t *>(block + off_kword(tau, 2 * q)) = wa;
                *reinterpret_cast<uint32_t *>(block + off_kword(tau, 2 * q + 1)) = wb;
                *reinterpret_cast<uint32_t *>(block + off_kmeta(tau, q)) = meta;
            } else {
                *reinterpret_cast<uint16_t *>(block + off_vpiece(tau, 4 * q)) = (uint16_t)wa;
                *reinterpret_cast<uint16_t *>(block + off_vpiece(tau, 4 * q + 1)) = (uint16_t)(wa >> 16);
                *reinterpret_cast<uint16_t *>(block + off_vpiece(tau, 4 * q + 2)) = (uint16_t)wb;
                *reinterpret_cast<uint16_t *>(block + off_vpiece(tau, 4 * q + 3)) = (uint16_t)(wb >> 16);
                *reinterpret_cast<uint32_t *>(block + off_vmeta(tau, q)) = meta;
            }
        }
    }
    __syncthreads();
    // the whole blocks, 48 x 16 bytes each (32 of codes, 16 of metadata)
    if (L0 >= 0) {
        const int first = (P0 + BLK_TOK - 1) / BLK_TOK, last = P1 / BLK_TOK;   // [first, last)
        const int i = threadIdx.x, k = i / 48, j = i % 48;
        if (first + k < last) {
            const int lb = first + k;
            const long long bi = cache_block_index(c.table, c.num_blocks, c.nblk, c.Hkv, b, h, lb);
            if (bi < 0) {
                if (j == 0) set_status(c.status, KVQ_DEV_BAD_TABLE);
            } else {
                const int off = j < 32 ? (kind == 0 ? 0 : OFF_VC) + 16 * j
                                       : (kind == 0 ? OFF_KM : OFF_VM) + 16 * (j - 32);
                *reinterpret_cast<uint4 *>(c.blocks + (size_t)bi * BLK_BYTES + off) =
                    *reinterpret_cast<const uint4 *>(&tile[lb - lb0][off]);
            }
        }
    }
    append_done(c);
}

// ---- pre-RoPE grouped-head key rotation ----------------------------------------------------------
// "RotateKV", abstract item (ii): the keys are rotated before RoPE, by one
// rotation across a group of GH consecutive KV heads.  The group's pre-RoPE
// keys (n = 128*GH channels, contiguous in K) are reordered by the group's
// permutation and transformed by an n-point FWHT / sqrt(n); each head's
// 128-channel slice is quantized into its own cache unit.  Values are
// rotated per head as in FWHT mode.  A sink keeps its key as given (fp16,
// pre-RoPE: the decode turns it by RoPE at its position) and its rotated
// value.  One warp per row: rows [0, nk) are key
// groups (b, t, group), rows [nk, nk + nv) value rows (b, t, h).  Lane l
// holds the group elements j*128 + 4l + k (j < GH, k < 4): the FWHT stages
// over k and l are fwht128_warp's, the ones over j run in registers (the
// Sylvester transform is a product of commuting butterfly stages, one per
// index bit, so their order does not matter).
struct PreRopeRows {
    const uint16_t *K, *V;     // cache: [B][T][Hkv][128]; debug: K = X [N][128*GH]
    const int32_t *perm;       // cache: [2][Hkv*128] (plane 0 key groups, plane 1 value
                               // heads); debug: one group permutation [128*GH]
    float *out_f32;            // debug output [N][128*GH] or nullptr
    long long nk, nv;          // cache: B*T*(Hkv/GH) key-group rows, B*T*Hkv value rows
};

template <int GH>
__device__ __forceinline__ float inv_sqrt_group() {
    return GH == 1 ? 0.08838834764831845f
                   : (GH == 2 ? 0.0625f : (GH == 4 ? 0.04419417382415922f : 0.03125f));
}

template <int GH, bool TO_CACHE>
__global__ void __launch_bounds__(FWHT_THREADS) append_prerope_kernel(PreRopeRows a, CacheDst c) {
    constexpr int n = GH * D;
    __shared__ __align__(16) uint16_t xs[FWHT_THREADS / 32][n];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_trigger();
    const long long row = (long long)blockIdx.x * (FWHT_THREADS / 32) + warp;
    if (row < a.nk + a.nv) {
        const bool key = row < a.nk;
        int b = 0, t = 0, hh = 0, L0 = 0;
        if (TO_CACHE) {
            const int nper = key ? c.Hkv / GH : c.Hkv;     // groups (keys) or heads (values)
            long long r2 = key ? row : row - a.nk;
            hh = (int)(r2 % nper);
            r2 /= nper;
            t = (int)(r2 % c.T);
            b = (int)(r2 / c.T);
            L0 = start_len_thread(c, b, key && lane == 0 && t == 0 && hh == 0);
        }
        if (L0 >= 0 && key) {
            const uint16_t *src = TO_CACHE
                                      ? a.K + (((size_t)b * c.T + t) * c.Hkv + (size_t)hh * GH) * D
                                      : a.K + (size_t)row * n;
            const int32_t *pg = TO_CACHE ? a.perm + (size_t)hh * n : a.perm;
#pragma unroll
            for (int j = 0; j < GH; j++)
                *reinterpret_cast<uint2 *>(&xs[warp][j * D + 4 * lane]) =
                    *reinterpret_cast<const uint2 *>(src + j * D + 4 * lane);
            __syncwarp();
            float v[GH][4];
#pragma unroll
            for (int j = 0; j < GH; j++) {
                const int4 pi = *reinterpret_cast<const int4 *>(pg + j * D + 4 * lane);
                v[j][0] = __half2float(__ushort_as_half(xs[warp][pi.x & (n - 1)]));
                v[j][1] = __half2float(__ushort_as_half(xs[warp][pi.y & (n - 1)]));
                v[j][2] = __half2float(__ushort_as_half(xs[warp][pi.z & (n - 1)]));
                v[j][3] = __half2float(__ushort_as_half(xs[warp][pi.w & (n - 1)]));
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
            const float sc = inv_sqrt_group<GH>();
#pragma unroll
            for (int j = 0; j < GH; j++) {
#pragma unroll
                for (int k = 0; k < 4; k++) v[j][k] *= sc;
                if (TO_CACHE)
                    cache_epilogue(c, b, t, hh * GH + j, 0, L0, v[j], &xs[warp][j * D + 4 * lane]);
                else
                    *reinterpret_cast<float4 *>(a.out_f32 + (size_t)row * n + j * D + 4 * lane) =
                        make_float4(v[j][0], v[j][1], v[j][2], v[j][3]);
            }
        } else if (L0 >= 0 && TO_CACHE) {
            // a value row: per-head permutation + 128-point FWHT
            const uint16_t *src = a.V + (((size_t)b * c.T + t) * c.Hkv + hh) * D;
            const int32_t *pv = a.perm + ((size_t)c.Hkv + hh) * D;
            *reinterpret_cast<uint2 *>(&xs[warp][4 * lane]) =
                *reinterpret_cast<const uint2 *>(src + 4 * lane);
            const int4 pi = *reinterpret_cast<const int4 *>(pv + 4 * lane);
            __syncwarp();
            float v[4];
            v[0] = __half2float(__ushort_as_half(xs[warp][pi.x & (D - 1)]));
            v[1] = __half2float(__ushort_as_half(xs[warp][pi.y & (D - 1)]));
            v[2] = __half2float(__ushort_as_half(xs[warp][pi.z & (D - 1)]));
            v[3] = __half2float(__ushort_as_half(xs[warp][pi.w & (D - 1)]));
            fwht128_warp(v);
#pragma unroll
            for (int k = 0; k < 4; k++) v[k] *= 0.08838834764831845f;
            cache_epilogue(c, b, t, hh, 1, L0, v);
        }
    }
    if (TO_CACHE) append_done(c);
}

template <int GH>
static cudaError_t launch_prerope_t(const PreRopeRows &a, const CacheDst &c, bool to_cache,
                                    cudaStream_t st) {
    const long long rows = a.nk + a.nv;
    const unsigned grid = (unsigned)((rows + FWHT_THREADS / 32 - 1) / (FWHT_THREADS / 32));
    if (to_cache)
        return launch_pdl(append_prerope_kernel<GH, true>, dim3(grid), dim3(FWHT_THREADS), 0, st,
                          a, c);
    append_prerope_kernel<GH, false><<<grid, FWHT_THREADS, 0, st>>>(a, c);
    return cudaGetLastError();
}

static cudaError_t launch_prerope(int gh, const PreRopeRows &a, const CacheDst &c, bool to_cache,
                                  cudaStream_t st) {
    switch (gh) {
        case 1: return launch_prerope_t<1>(a, c, to_cache, st);
        case 2: return launch_prerope_t<2>(a, c, to_cache, st);
        case 4: return launch_prerope_t<4>(a, c, to_cache, st);
        case 8: return launch_prerope_t<8>(a, c, to_cache, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_append_prerope(const uint16_t *K, const uint16_t *V, int T, int gh,
                                  const int32_t *perm, const kvq_cache_desc &cd,
                                  int32_t *seq_lens, cudaStream_t st) {
    const CacheDst c = cache_dst(cd, seq_lens, T);
    PreRopeRows a;
    a.K = K;
    a.V = V;
    a.perm = perm;
    a.out_f32 = nullptr;
    a.nk = (long long)cd.B * T * (cd.Hkv / gh);
    a.nv = (long long)cd.B * T * cd.Hkv;
    return launch_prerope(gh, a, c, true, st);
}

cudaError_t launch_debug_rotate_group(const uint16_t *X, int N, int gh, const int32_t *perm,
                                     float *out, cudaStream_t st) {
    CacheDst c{};
    PreRopeRows a;
    a.K = a.V = X;
    a.perm = perm;
    a.out_f32 = out;
    a.nk = N;
    a.nv = 0;
    return launch_prerope(gh, a, c, false, st);
}

// ---- quantizer test export ---------------------------------------------------------------------
__global__ void debug_quantize_kernel(const float *X, int N, uint8_t *codes, uint16_t *meta) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
    if (row >= N) return;
    const float4 x4 = *reinterpret_cast<const float4 *>(X + row * D + 4 * lane);
    const float v[4] = {x4.x, x4.y, x4.z, x4.w};
    const QuantWord q = quantize_row_warp(v);
    if (lane < 8) *reinterpret_cast<uint32_t *>(codes + row * 32 + 4 * lane) = q.word;
    if ((lane & 7) == 0) {
        const int g = lane >> 3;
        meta[(row * NG + g) * 2] = q.s;
        meta[(row * NG + g) * 2 + 1] = q.z;
    }
}

// ---- sink identification ------------------------------------------------------------------
// One CTA per sequence.  The sinks are the tokens whose activations are
// massive ("RotateKV", abstract item (iii)): token t of the T about to be
// appended is one when act[b][t] >= tau, and the sequence's free fp16 rows
// go to such tokens in position order.  Tokens go in passes of up to
// ID_THREADS * 32: thread i flags a contiguous run of at most 32 tokens in a
// bit mask, an exclusive scan of the flag counts over the CTA ranks the
// flagged tokens, and each thread writes the positions whose rank is below
// the number of rows.
constexpr int ID_THREADS = 1024;
constexpr int ID_RUN = 32;

__global__ void __launch_bounds__(ID_THREADS)
    identify_sinks_kernel(const float *act, int T, float tau, CacheDst c) {
    __shared__ int wsum[ID_THREADS / 32];
    const int b = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_wait();
    pdl_trigger();
    const int L0 = c.seq_lens[b];
    // a sequence the append skips (and flags) gets no sinks
    if (L0 < 0 || (long long)L0 + T > c.capacity) return;
    int cnt = min(max(c.sink_count[b], 0), c.S);
    const float *ab = act + (size_t)b * T;
    for (int pass0 = 0; pass0 < T && cnt < c.S; pass0 += ID_THREADS * ID_RUN) {
        const int n = min(T - pass0, ID_THREADS * ID_RUN);
        const int run = (n + ID_THREADS - 1) / ID_THREADS;        // <= ID_RUN
        const int lo = pass0 + threadIdx.x * run;
        const int hi = min(lo + run, pass0 + n);
        uint32_t mask = 0;
        for (int t = lo; t < hi; t++)
            if (ab[t] >= tau) mask |= 1u << (t - lo);
        const int k = __popc(mask);
        int incl = k;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll 4
        for (int w = 0; w < ID_THREADS / 32; w++) {
            const int x = wsum[w];
            before += w < warp ? x : 0;
            total += x;
        }
        int rank = cnt + before + incl - k;
        while (mask != 0u && rank < c.S) {
            const int i = __ffs(mask) - 1;
            mask &= mask - 1u;
            c.sink_pos[(size_t)b * c.S + rank] = L0 + lo + i;
            ++rank;
        }
        cnt = min(c.S, cnt + total);
        __syncthreads();                                   // wsum is rewritten next pass
    }
    if (threadIdx.x == 0) c.sink_count[b] = cnt;
}

cudaError_t launch_identify_sinks(const float *act, int T, float tau, const kvq_cache_desc &cd,
                                  const int32_t *seq_lens, cudaStream_t st) {
    const CacheDst c = cache_dst(cd, const_cast<int32_t *>(seq_lens), T);   // seq_lens only read
    return launch_pdl(identify_sinks_kernel, dim3(cd.B), dim3(ID_THREADS), 0, st, act, T, tau, c);
}

// ---- host launchers (called from kvq_api.cu) -----------------------------------------------------
cudaError_t launch_append_small(const uint16_t *K, const uint16_t *V, int T, int mode,
                                const float *R_k, const float *R_v, const int32_t *perm,
                                const kvq_cache_desc &cd, int32_t *seq_lens,
                                cudaStream_t st) {
    const CacheDst c = cache_dst(cd, seq_lens, T);
    if (mode == KVQ_ROT_DENSE) {
        DenseRows a;
        a.X0 = K;
        a.X1 = V;
        a.R0 = R_k;
        a.R1 = R_v;
        a.out_f32 = nullptr;
        a.n_rows = 0;
        a.tchunk = T <= 64 ? T : 64;
        // fewer than DENSE_BATCH tokens: one CTA takes several sequences
        a.bpc = T >= DENSE_BATCH ? 1 : std::min(cd.B, DENSE_BATCH / T);
        dim3 grid((T + a.tchunk - 1) / a.tchunk, cd.Hkv, 2 * ((cd.B + a.bpc - 1) / a.bpc));
        return launch_pdl(append_dense_kernel<true>, grid, dim3(DENSE_THREADS), 0, st, a, c);
    } else {
        FwhtRows a;
        a.X0 = K;
        a.X1 = V;
        a.perm = perm;
        a.out_f32 = nullptr;
        a.n_rows = (long long)cd.B * T * cd.Hkv * 2;
        if (T >= FWHT_CHUNK_MIN_T)
            return launch_pdl(append_fwht_chunk_kernel,
                              dim3((T + FWHT_ROWS - 1) / FWHT_ROWS, 2 * cd.Hkv, cd.B),
                              dim3(FWHT_THREADS), 0, st, a, c);
        return launch_pdl(append_fwht_kernel<true>,
                          dim3((unsigned)((long long)cd.B * T), (2 * cd.Hkv + FWHT_ROWS - 1) / FWHT_ROWS),
                          dim3(FWHT_THREADS), 0, st, a, c);
    }
}

cudaError_t launch_debug_rotate_small(const uint16_t *X, int N, int mode, const float *R,
                                      const int32_t *perm, float *out, cudaStream_t st) {
    CacheDst c{};
    if (mode == KVQ_ROT_DENSE) {
        DenseRows a;
        a.X0 = a.X1 = X;
        a.R0 = a.R1 = R;
        a.out_f32 = out;
        a.n_rows = N;
        a.tchunk = 64;
        a.bpc = 1;
        append_dense_kernel<false><<<(N + 63) / 64, DENSE_THREADS, 0, st>>>(a, c);
    } else {
        FwhtRows a;
        a.X0 = a.X1 = X;
        a.perm = perm;
        a.out_f32 = out;
        a.n_rows = N;
        append_fwht_kernel<false><<<(N + FWHT_ROWS - 1) / FWHT_ROWS, FWHT_THREADS, 0, st>>>(a, c);
    }
    return cudaGetLastError();
}

cudaError_t launch_debug_quantize(const float *X, int N, uint8_t *codes, uint16_t *meta,
                                  cudaStream_t st) {
    debug_quantize_kernel<<<(N + 7) / 8, 256, 0, st>>>(X, N, codes, meta);
    return cudaGetLastError();
}

}  // namespace kvq
