// moe_tc.cu -- the grouped gate/up and down stages for >= 32 tokens per step on the fifth
// generation tensor cores (tcgen05.mma kind::i8, accumulators in tensor memory), sm_100a.
//
// At 32 or more tokens the selected experts each serve a few tokens ("iPhone Runs a 20B Model at
// 120 tok/s", "What Makes 120 tok/s So Fast?": batched work turns the matrix-vector products of
// decode into small matrix products), so every expert's rows are decoded once and multiplied
// against all of its tokens at once.  One CTA per (distinct expert, 128 rows) for gate/up, and per
// (distinct expert, 2 x 128 rows) for down, whose short K (f) lets it stage the B rows of the
// whole K once per pass for both row blocks.  160 threads:
//   * four decoder warps, thread = row: per K-tile of 64 codes each thread decodes its row's 16
//     packed bytes by integer logic into int8 lanes of 64 * w (the table-free decode of
//     decode.cuh, position-major order) and writes them into shared memory in the tensor core's
//     K-major layout.  Beside them go the B rows: every activation limb of every token of the
//     pass (the expert's entries), put into the same order by a byte transpose.  Each thread
//     keeps the global loads of the next kTcDepth tiles in flight, and decoding runs ahead of the
//     tensor core by kTcStages buffers;
//   * one MMA warp: its lane 0 waits for a buffer's decoders (mbarrier), issues one MMA per
//     matrix and K step (M = 128, K = 32, N = the pass's B rows rounded up to 16; A = the weights,
//     signed int8) and commits to the buffer's second mbarrier, which frees it for the decoders.
//     With bf16 activations the three limbs of a token are three B rows, all unsigned: the hi
//     limb carries an offset of 128, and a row of ones gives the weights' row sums that take it
//     out again;
//   * the epilogue reads the accumulators with tcgen05.ld (thread = row), divides out the 64
//     exactly and recombines the limbs in int64, S = hi * 65536 + mid * 256 + lo: the same
//     integers as the dp4a and mma.sync kernels, so the outputs are identical.
// Every wait is bounded; after a timeout (status set) both sides keep the barrier protocol but
// skip their work, so no thread is left waiting.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "tern_common.cuh"
#include "tma.cuh"

namespace tern {

constexpr int kTcM = 128;        // rows per CTA (the MMA's M)
constexpr int kTcKT = 64;        // codes per K-tile: one 16-byte packed word per row
constexpr int kTcBRows = 64;     // rows of the B operand (limb rows of the pass's tokens): the largest N
constexpr int kTcBChunks = kTcBRows * (kTcKT / 16);  // 16-byte chunks of B per tile
constexpr int kTcDec = 128;      // decoder threads (thread = row); warp w reads accumulator lanes 32w .. 32w + 31
constexpr int kTcThreads = kTcDec + 32;  // and the MMA warp
constexpr int kTcStages = 2;     // operand buffers: 40 KB of shared memory per gate/up CTA
constexpr int kTcDepth = 4;      // K-tiles of global loads in flight per decoder thread
constexpr int kTcDownRB = 2;     // blocks of 128 rows per down CTA
constexpr int kTcBWholeMax = 512;  // largest K whose whole B operand (64 rows) a down CTA stages once per pass
constexpr int kTcABytes = kTcM * kTcKT;
constexpr int kTcBBytes = kTcBRows * kTcKT;
// Tokens per pass.  One int8 limb (int8 activations, signed): one B row per token.  Three limbs
// (bf16 activations): limb l of token n is B row l * NBp + n (NBp = the pass's tokens rounded up
// to 4), and row 3 * NBp is all ones: it accumulates the row sums of the weights, which turn
// the hi limb stored with an offset of 128 (so that every B row is unsigned) back into the signed
// limb.  So one MMA per matrix and K step covers every limb of every token of the pass, and the
// tensor core reads each weight tile from shared memory once.
template <int NL>
constexpr int kTcTokens() { return NL == 1 ? kTcBRows : (kTcBRows - 1) / 3 / 4 * 4; }
constexpr long long kTcWaitNs = 1000000000ll;

// K-major operand without swizzle: 8 rows x 16 bytes make a contiguous 128-byte core matrix,
// core matrices K-chunk-minor: byte `b` of row `r` of a tile is at
// ((r / 8) * (KT / 16) + b / 16) * 128 + (r % 8) * 16 + b % 16.  The MMA over bytes 32s .. 32s + 31
// starts at 2s * 128; the next 16 bytes of K are 128 bytes on (leading byte offset), the next 8
// rows (KT / 16) * 128 bytes on (stride byte offset).
__device__ __forceinline__ uint32_t tc_off(int r, int b) {
    return (uint32_t)((((r >> 3) * (kTcKT / 16) + (b >> 4)) << 7) + ((r & 7) << 4) + (b & 15));
}

// shared-memory matrix descriptor: start >> 4 in bits 0-13, leading byte offset >> 4 in bits
// 16-29, stride byte offset >> 4 in bits 32-45, version 1 in bits 46-47, base offset 0, layout
// type 0 (no swizzle) in bits 61-63
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr, uint32_t sbo_bytes = (kTcKT / 16) * 128) {
    const uint64_t lbo = 128u, sbo = sbo_bytes;
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFull) << 16) | (((sbo >> 4) & 0x3FFFull) << 32) |
           (1ull << 46);
}

// instruction descriptor: s32 accumulators (bits 4-5 = 2), A signed 8-bit (bits 7-9 = 1), B
// signed (1) or unsigned (0) 8-bit (bits 10-12), both K-major (bits 15, 16 = 0), N / 8 in bits
// 17-22, M / 16 in bits 24-28
__device__ __forceinline__ uint32_t tc_idesc(bool b_signed, int n) {
    return (2u << 4) | (1u << 7) | ((b_signed ? 1u : 0u) << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kTcM >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t dtmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(dtmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_ld4(uint32_t taddr, uint32_t (&v)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_alloc(uint32_t *dst, uint32_t ncols) {  // one full warp
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {  // the same warp
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// One K-tile of global data for a decoder thread: the packed 16 bytes (64 codes) of row
// threadIdx.x of each matrix, and two of the tile's B chunks (chunk i = threadIdx.x + j * kTcDec:
// B row i % 64, 16-byte chunk i / 64 of the tile).
constexpr int kTcBPer = kTcBChunks / kTcDec;

// BW: the B operand of the whole K is staged once per pass instead (tiles carry no B chunks)
template <int NM, bool BW>
struct TcTile {
    uint4 a[NM];
    uint4 b[BW ? 1 : kTcBPer];
};

// Where a decoder thread's data of tile 0 sits.  A CTA takes NRB blocks of 128 rows one after
// another, ntk K-tiles each: tile t is K-tile t % ntk of row block t / ntk, t % ntk uint4 into the
// row and rbstep uint4 on per row block; for the limbs 4 (t % ntk) uint4 on.  A null pointer, or
// a row block at or past nrb (the blocks in which this thread's row exists), reads as zero.  Each
// B chunk is then XORed with bx[j]: 0x80 in every byte of a hi limb (the offset of 128), 0x01 in
// every byte of the ones row.
// row block of tile t (ntk tiles per block)
template <int NRB>
__device__ __forceinline__ int tc_rb(int t, int ntk) {
    return NRB == 1 ? 0 : (NRB == 2 ? (t >= ntk ? 1 : 0) : t / ntk);
}

template <int NM>
struct TcSrc {
    const uint4 *a[NM];
    const uint4 *b[kTcBPer];
    uint32_t bx[kTcBPer];
    int64_t rbstep;
    int ntk, nrb;
};

// B rows of a pass of nb tokens with NL limbs, and its MMA's N (a multiple of 16)
template <int NL>
__device__ __forceinline__ int tc_nbp(int nb) { return NL == 1 ? nb : (nb + 3) & ~3; }
template <int NL>
__device__ __forceinline__ int tc_n(int nb) {
    const int rows = NL == 1 ? nb : 3 * tc_nbp<NL>(nb) + 1;
    return (rows + 15) & ~15;
}

// mats[m]: row 0 of the CTA's first row block; nrows: the CTA's rows that exist (from row 0 on)
template <int NM, int NL, int NRB>
__device__ __forceinline__ void tc_src(TcSrc<NM> &p, const uint8_t *const (&mats)[NM], int64_t rowb, int nrows,
                                       int ntk, const uint32_t *__restrict__ src, int K4,
                                       const int32_t *__restrict__ ent, int q0, int nb, int div) {
    const int r = threadIdx.x;
#pragma unroll
    for (int m = 0; m < NM; m++)
        p.a[m] = r < nrows ? reinterpret_cast<const uint4 *>(mats[m] + (int64_t)r * rowb) : nullptr;
    p.rbstep = (int64_t)kTcM * rowb / 16;
    p.ntk = ntk;
    p.nrb = r < nrows ? min(NRB, (nrows - r + kTcM - 1) / kTcM) : 0;
    const int nbp = tc_nbp<NL>(nb);
#pragma unroll
    for (int j = 0; j < kTcBPer; j++) {
        const int i = threadIdx.x + j * kTcDec;
        const int row = i % kTcBRows, c = i / kTcBRows;
        int l = 0, n = row;
        if (NL > 1) {
            l = row / nbp;
            n = row - l * nbp;
        }
        p.b[j] = nullptr;
        p.bx[j] = 0u;
        if (l < NL && n < nb) {
            const int64_t vec = ent[q0 + n] / div;
            p.b[j] = reinterpret_cast<const uint4 *>(src + (vec * NL + l) * K4) + c;
            if (NL > 1 && l == 0) p.bx[j] = 0x80808080u;
        } else if (NL > 1 && row == 3 * nbp) {
            p.bx[j] = 0x01010101u;
        }
    }
}

template <int NM, int NRB, bool BW>
__device__ __forceinline__ void tc_load(TcTile<NM, BW> &p, const TcSrc<NM> &q, int t) {
    const int rb = tc_rb<NRB>(t, q.ntk), kt = t - rb * q.ntk;
#pragma unroll
    for (int m = 0; m < NM; m++)
        p.a[m] = rb < q.nrb ? __ldg(q.a[m] + rb * q.rbstep + kt) : make_uint4(0u, 0u, 0u, 0u);
    if (BW) return;
#pragma unroll
    for (int j = 0; j < kTcBPer; j++) {
        const uint4 v = q.b[j] ? __ldg(q.b[j] + (kTcKT / 16) * kt) : make_uint4(0u, 0u, 0u, 0u);
        p.b[j] = make_uint4(v.x ^ q.bx[j], v.y ^ q.bx[j], v.z ^ q.bx[j], v.w ^ q.bx[j]);
    }
}

// The tile into one operand buffer.  Packed word q of the row (codes 16q .. 16q + 15) becomes
// 16-byte chunk q of the row in the table-free decode's position-major order: byte 4j + b
// holds 64 times the weight of code 16q + 4b + j (decode.cuh).  The B chunks take the same
// order by a 4x4 byte transpose, so A and B agree on every K index of the tile.
template <int NM, bool BW>
__device__ __forceinline__ void tc_store(const TcTile<NM, BW> &p, unsigned char *A, unsigned char *B) {
    const int r = threadIdx.x;
#pragma unroll
    for (int m = 0; m < NM; m++) {
        const uint32_t pw[4] = {p.a[m].x, p.a[m].y, p.a[m].z, p.a[m].w};
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const uint32_t sf = tern_signed_fields(pw[q]);
            *reinterpret_cast<uint4 *>(A + (size_t)m * kTcABytes + tc_off(r, 16 * q)) =
                make_uint4(tern_position_lanes(sf, 0), tern_position_lanes(sf, 1), tern_position_lanes(sf, 2),
                           tern_position_lanes(sf, 3));
        }
    }
    if (BW) return;
#pragma unroll
    for (int j = 0; j < kTcBPer; j++) {
        const int i = threadIdx.x + j * kTcDec;
        uint4 v;
        bytes_transpose4(p.b[j].x, p.b[j].y, p.b[j].z, p.b[j].w, v.x, v.y, v.z, v.w);
        *reinterpret_cast<uint4 *>(B + tc_off(i % kTcBRows, 16 * (i / kTcBRows))) = v;
    }
}

// The B operand of the whole K (kb bytes per row) for one pass, in the K-major layout with a
// stride of kb / 16 core matrices between 8-row groups.  B row r is staged by threads r and r + 64
// (chunk i = threadIdx.x + j * kTcDec keeps row threadIdx.x % 64 for every j): chunk c = c0 + 2j
// of the row, c0 = threadIdx.x / 64, from the pointer tc_src set for j = 0.
template <int NM>
__device__ __forceinline__ void tc_stage_b_whole(const TcSrc<NM> &q, unsigned char *B, int kb) {
    const int row = threadIdx.x % kTcBRows, c0 = threadIdx.x / kTcBRows;
    const int nch = kb / 32;  // chunks of this thread
    const uint32_t x = q.bx[0];
    for (int j0 = 0; j0 < nch; j0 += 8) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; u++)
            v[u] = (q.b[0] && j0 + u < nch) ? __ldg(q.b[0] + 2 * (j0 + u)) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 8; u++) {
            if (j0 + u >= nch) continue;
            const int c = c0 + 2 * (j0 + u);
            uint4 w;
            bytes_transpose4(v[u].x ^ x, v[u].y ^ x, v[u].z ^ x, v[u].w ^ x, w.x, w.y, w.z, w.w);
            *reinterpret_cast<uint4 *>(B + ((((row >> 3) * (kb / 16) + c) << 7) + ((row & 7) << 4))) = w;
        }
    }
}

// Shared state of one CTA's pipeline: operand buffers, their mbarriers and the tile counter.
// Tile g (counted over the CTA's passes) goes to buffer g % kTcStages as that buffer's use
// g / kTcStages.  mb_full[b] completes a phase when the four decoder warps have stored a tile
// into buffer b; mb_done[b] when the MMAs reading it have finished (tcgen05.commit).
struct TcPipe {
    unsigned char *A, *B;
    uint64_t *full, *done;
    uint32_t tmem;
    unsigned it;
    bool failed;  // a wait timed out (status set): the pipeline keeps its protocol but skips work
};

// Decoder side of one pass (warps 0..3): tiles 0 .. ntile-1 of the pass, kTcDepth tiles of global
// loads in flight, each tile decoded into the next buffer once the tensor core has finished with
// that buffer's previous tile.  Returns once every MMA of the pass has completed.
template <int NM, int NRB, bool BW>
__device__ __forceinline__ void tc_decode_pass(TcPipe &pp, const TcSrc<NM> &src, int ntile, int kb, int *status) {
    const int lane = threadIdx.x & 31;
    TcTile<NM, BW> buf[kTcDepth];
#pragma unroll
    for (int j = 0; j < kTcDepth; j++)
        if (j < ntile) tc_load<NM, NRB, BW>(buf[j], src, j);
    // the whole B while the first tiles' loads are in flight; the previous pass's MMAs are done
    if (BW) tc_stage_b_whole<NM>(src, pp.B, kb);
    for (int t0 = 0; t0 < ntile; t0 += kTcDepth) {
#pragma unroll
        for (int j = 0; j < kTcDepth; j++) {
            const int t = t0 + j;
            if (t < ntile) {
                const unsigned g = pp.it + (unsigned)t;
                const int b = (int)(g % kTcStages);
                if (g >= kTcStages && !pp.failed &&
                    !mbar_wait_sleep(&pp.done[b], ((g / kTcStages) - 1u) & 1u, kTcWaitNs, status))
                    pp.failed = true;
                if (!pp.failed)
                    tc_store<NM, BW>(buf[j], pp.A + (size_t)b * NM * kTcABytes, pp.B + (size_t)b * kTcBBytes);
                if (t + kTcDepth < ntile) tc_load<NM, NRB, BW>(buf[j], src, t + kTcDepth);
                fence_async_smem();  // the generic-proxy stores above, visible to the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(&pp.full[b]);
            }
        }
    }
    const unsigned last = pp.it + (unsigned)ntile - 1u;
    if (!pp.failed && !mbar_wait_sleep(&pp.done[last % kTcStages], (last / kTcStages) & 1u, kTcWaitNs, status))
        pp.failed = true;
    tc_fence_after();
    pp.it += (unsigned)ntile;
}

// MMA side of one pass (lane 0 of warp 4): per tile, wait for the decoders, issue NM x (kTcKT /
// 32) MMAs (M = 128, N = n, K = 32) into accumulator columns (rb * NM + m) * kTcBRows .. + n of
// the tile's row block rb, and commit to the buffer's mbarrier.  The descriptors of buffer 0 are
// built once; a buffer, matrix or K step is an offset added to the start-address field.
template <int NM, int NRB, bool BW>
__device__ __forceinline__ void tc_mma_pass(TcPipe &pp, int ntile, int ntk, int kb, uint32_t idesc, int *status) {
    const uint64_t a0 = tc_desc(smem_u32(pp.A)), b0 = tc_desc(smem_u32(pp.B), BW ? (uint32_t)(kb / 16) * 128u : (kTcKT / 16) * 128u);
    for (int t = 0; t < ntile; t++) {
        const unsigned g = pp.it + (unsigned)t;
        const int b = (int)(g % kTcStages);
        const int rb = tc_rb<NRB>(t, ntk), kt = t - rb * ntk;
        if (!pp.failed && !mbar_wait_sleep(&pp.full[b], (g / kTcStages) & 1u, kTcWaitNs, status)) pp.failed = true;
        tc_fence_after();
        if (!pp.failed) {
#pragma unroll
            for (int s = 0; s < kTcKT / 32; s++)
#pragma unroll
                for (int m = 0; m < NM; m++)
                    tc_mma(pp.tmem + (uint32_t)((rb * NM + m) * kTcBRows),
                           a0 + (uint64_t)((((b * NM + m) * kTcABytes) + s * 256) >> 4),
                           b0 + (uint64_t)((BW ? (kt * (kTcKT / 16) + 2 * s) * 128 : (b * kTcBBytes) + s * 256) >> 4),
                           idesc, (kt > 0 || s > 0) ? 1u : 0u);
        }
        tc_commit(&pp.done[b]);
    }
    pp.it += (unsigned)ntile;
}

// The CTA's set-up: mbarriers, tensor memory (warp 0), then one barrier.
__device__ __forceinline__ void tc_setup(TcPipe &pp, unsigned char *smem, int a_bytes, uint64_t *full, uint64_t *done,
                                         uint32_t *s_tmem, uint32_t ncols) {
    pp.A = smem;
    pp.B = smem + a_bytes;
    pp.full = full;
    pp.done = done;
    pp.it = 0;
    pp.failed = false;
    if (threadIdx.x == 0) {
        for (int b = 0; b < kTcStages; b++) {
            mbar_init(&full[b], kTcDec / 32);
            mbar_init(&done[b], 1);
        }
        fence_mbar_init();
    }
    if (threadIdx.x < 32) tc_alloc(s_tmem, ncols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pp.tmem = *s_tmem;
}

// The end: the MMA thread waits for its last commit, then warp 0 frees the tensor memory.
__device__ __forceinline__ void tc_teardown(TcPipe &pp, uint32_t ncols, int *status) {
    if (threadIdx.x == kTcDec && pp.it > 0 && !pp.failed) {
        const unsigned last = pp.it - 1u;
        mbar_wait(&pp.done[last % kTcStages], (last / kTcStages) & 1u, kTcWaitNs, status);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x < 32) tc_dealloc(pp.tmem, ncols);
}

// an accumulator column read back: 64 times the exact sum (the weights are 64 * w)
__device__ __forceinline__ long long tc_acc(uint32_t v) { return (long long)((int32_t)v >> 6); }

// The exact integer sums of tokens n0 .. n0 + 3 (pass of nbp B rows per limb) for the matrix
// whose accumulators start at column `col` of this thread's lane: three limbs recombined, the
// hi limb's offset of 128 taken out with the row sum R of the ones row.
template <int NL>
__device__ __forceinline__ void tc_sums4(uint32_t ta, int col, int nbp, int n0, long long R, long long (&S)[4]) {
    if (NL == 1) {
        uint32_t v[4];
        tc_ld4(ta + (uint32_t)(col + n0), v);
        tc_wait_ld();
#pragma unroll
        for (int z = 0; z < 4; z++) S[z] = tc_acc(v[z]);
    } else {
        uint32_t v0[4], v1[4], v2[4];
        tc_ld4(ta + (uint32_t)(col + n0), v0);
        tc_ld4(ta + (uint32_t)(col + nbp + n0), v1);
        tc_ld4(ta + (uint32_t)(col + 2 * nbp + n0), v2);
        tc_wait_ld();
#pragma unroll
        for (int z = 0; z < 4; z++) S[z] = (tc_acc(v0[z]) - 128 * R) * 65536 + tc_acc(v1[z]) * 256 + tc_acc(v2[z]);
    }
}

// row sum of the weights over K (the ones row of a three-limb pass), for the matrix at `col`
template <int NL>
__device__ __forceinline__ long long tc_rowsum(uint32_t ta, int col, int nbp) {
    if (NL == 1) return 0;
    uint32_t v[4];
    tc_ld4(ta + (uint32_t)(col + 3 * nbp), v);
    tc_wait_ld();
    return tc_acc(v[0]);
}

// grid: (distinct experts bound, f / 128); 128 rows of gate and up per CTA
template <int NL>
__global__ void __launch_bounds__(kTcThreads, 3) gateup_tc_kernel(
    const uint8_t *__restrict__ gate, const uint8_t *__restrict__ up, const float *__restrict__ sg,
    const float *__restrict__ su, int d, int f, int k, const int32_t *__restrict__ n_unique,
    const int32_t *__restrict__ uexp, const int32_t *__restrict__ uoff, const int32_t *__restrict__ ent,
    const uint32_t *__restrict__ xw, const float *__restrict__ xsc, float *__restrict__ h,
    int32_t *__restrict__ acc_g, int32_t *__restrict__ acc_u, int *status) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t mb_full[kTcStages], mb_done[kTcStages];
    __shared__ uint32_t s_tmem;
    __shared__ int s_ent[2][kTcTokens<NL>()];
    __shared__ float s_sc[2][kTcTokens<NL>()];
    const int u = blockIdx.x;
    if (u >= *n_unique) return;  // before any tensor memory is held
    constexpr uint32_t ALLOC = 2 * kTcBRows;
    constexpr int NBMAX = kTcTokens<NL>();
    const int tid = threadIdx.x, warp = tid >> 5;
    const int e = uexp[u], e0 = uoff[u], e1 = uoff[u + 1];
    const int row0 = blockIdx.y * kTcM, nrows = min(kTcM, f - row0);
    const int64_t rowb = d / 4;
    const int ntile = d / kTcKT;
    const uint8_t *const mats[2] = {gate + ((int64_t)e * f + row0) * rowb, up + ((int64_t)e * f + row0) * rowb};
    TcPipe pp;
    tc_setup(pp, smem, kTcStages * 2 * kTcABytes, mb_full, mb_done, &s_tmem, ALLOC);
    for (int q0 = e0, pass = 0; q0 < e1; q0 += NBMAX, pass++) {
        const int nb = min(NBMAX, e1 - q0), nbp = tc_nbp<NL>(nb);
        if (warp == kTcDec / 32) {  // the MMA warp
            if ((tid & 31) == 0) tc_mma_pass<2, 1, false>(pp, ntile, ntile, d, tc_idesc(NL == 1, tc_n<NL>(nb)), status);
            continue;
        }
        // the pass's entries and activation scales, for the epilogue (two copies by pass parity:
        // a copy is written again only after every decoder thread has passed the barrier below
        // in the pass between)
        int *const te = s_ent[pass & 1];
        float *const tsc = s_sc[pass & 1];
        if (tid < nb) {
            te[tid] = ent[q0 + tid];
            tsc[tid] = xsc[te[tid] / k];
        }
        TcSrc<2> src;
        tc_src<2, NL, 1>(src, mats, rowb, nrows, ntile, xw, d / 4, ent, q0, nb, k);
        tc_decode_pass<2, 1, false>(pp, src, ntile, d, status);
        named_bar_sync(1, kTcDec);
        // thread = row of this tile; nb is the same in every thread, so the accumulator loads
        // stay collective
        const int j = row0 + tid;
        const uint32_t ta = pp.tmem + ((uint32_t)(32 * warp) << 16);
        const bool live = j < f && !pp.failed;
        const float sgv = live ? sg[(int64_t)e * f + j] : 0.0f, suv = live ? su[(int64_t)e * f + j] : 0.0f;
        const long long Rg = tc_rowsum<NL>(ta, 0, nbp), Ru = tc_rowsum<NL>(ta, kTcBRows, nbp);
#pragma unroll 1
        for (int n0 = 0; n0 < nb; n0 += 4) {
            long long Sg[4], Su[4];
            tc_sums4<NL>(ta, 0, nbp, n0, Rg, Sg);
            tc_sums4<NL>(ta, kTcBRows, nbp, n0, Ru, Su);
#pragma unroll
            for (int z = 0; z < 4; z++) {
                const int n = n0 + z;
                if (!live || n >= nb) continue;
                const int entry = te[n];
                const float xsv = tsc[n];
                float hv;
                if (NL == 1) {
                    acc_g[(int64_t)entry * f + j] = (int32_t)Sg[z];
                    acc_u[(int64_t)entry * f + j] = (int32_t)Su[z];
                    const float gv = __fmul_rn(__fmul_rn(__int2float_rn((int)Sg[z]), sgv), xsv);
                    const float uv = __fmul_rn(__fmul_rn(__int2float_rn((int)Su[z]), suv), xsv);
                    hv = swiglu_f32((double)gv, (double)uv);
                } else {
                    const int sh = __float_as_int(xsv);
                    hv = swiglu_f32(ldexp((double)Sg[z], -sh) * (double)sgv, ldexp((double)Su[z], -sh) * (double)suv);
                }
                h[(int64_t)entry * f + j] = hv;
            }
        }
        // every read of the accumulators done before this warp's next arrival lets the MMA
        // thread overwrite them
        tc_fence_before();
    }
    tc_teardown(pp, ALLOC, status);
}

// grid: (distinct experts bound, d / (128 kTcDownRB)); kTcDownRB blocks of 128 output rows per
// CTA, streamed as one run of tiles (the K of a down row is short: f / 64 tiles per block).  BW:
// the B rows of the whole K (f bytes each) staged once per pass, for f <= kTcBWholeMax; the row
// blocks then share them instead of restaging them per tile
template <int NL, bool BW>
__global__ void __launch_bounds__(kTcThreads, 4) down_tc_kernel(
    const uint8_t *__restrict__ down, const float *__restrict__ sd, int d, int f, const int32_t *__restrict__ n_unique,
    const int32_t *__restrict__ uexp, const int32_t *__restrict__ uoff, const int32_t *__restrict__ ent,
    const uint32_t *__restrict__ hw, const float *__restrict__ hsc, double *__restrict__ ye,
    int32_t *__restrict__ acc_d, int *status) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t mb_full[kTcStages], mb_done[kTcStages];
    __shared__ uint32_t s_tmem;
    __shared__ int s_ent[2][kTcTokens<NL>()];
    __shared__ float s_sc[2][kTcTokens<NL>()];
    const int u = blockIdx.x;
    if (u >= *n_unique) return;
    constexpr int NRB = kTcDownRB;
    constexpr uint32_t ALLOC = NRB * kTcBRows;
    constexpr int NBMAX = kTcTokens<NL>();
    const int tid = threadIdx.x, warp = tid >> 5;
    const int e = uexp[u], e0 = uoff[u], e1 = uoff[u + 1];
    const int row0 = blockIdx.y * NRB * kTcM, nrows = min(NRB * kTcM, d - row0);
    const int64_t rowb = f / 4;
    const int ntk = f / kTcKT, ntile = NRB * ntk;
    const uint8_t *const mats[1] = {down + ((int64_t)e * d + row0) * rowb};
    TcPipe pp;
    tc_setup(pp, smem, kTcStages * kTcABytes, mb_full, mb_done, &s_tmem, ALLOC);
    for (int q0 = e0, pass = 0; q0 < e1; q0 += NBMAX, pass++) {
        const int nb = min(NBMAX, e1 - q0), nbp = tc_nbp<NL>(nb);
        if (warp == kTcDec / 32) {
            if ((tid & 31) == 0) tc_mma_pass<1, NRB, BW>(pp, ntile, ntk, f, tc_idesc(NL == 1, tc_n<NL>(nb)), status);
            continue;
        }
        int *const te = s_ent[pass & 1];
        float *const tsc = s_sc[pass & 1];
        if (tid < nb) {
            te[tid] = ent[q0 + tid];
            tsc[tid] = hsc[te[tid]];
        }
        TcSrc<1> src;
        tc_src<1, NL, NRB>(src, mats, rowb, nrows, ntk, hw, f / 4, ent, q0, nb, 1);
        tc_decode_pass<1, NRB, BW>(pp, src, ntile, f, status);
        named_bar_sync(1, kTcDec);
        const uint32_t ta = pp.tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll 1
        for (int rb = 0; rb < NRB; rb++) {
            const int i = row0 + rb * kTcM + tid;
            const bool live = i < d && !pp.failed;
            const float sdv = live ? sd[(int64_t)e * d + i] : 0.0f;
            const int col = rb * kTcBRows;
            const long long R = tc_rowsum<NL>(ta, col, nbp);
#pragma unroll 1
            for (int n0 = 0; n0 < nb; n0 += 4) {
                long long S[4];
                tc_sums4<NL>(ta, col, nbp, n0, R, S);
#pragma unroll
                for (int z = 0; z < 4; z++) {
                    const int n = n0 + z;
                    if (!live || n >= nb) continue;
                    const int entry = te[n];
                    const float hs = tsc[n];
                    double v;
                    if (NL == 1) {
                        acc_d[(int64_t)entry * d + i] = (int32_t)S[z];
                        v = (double)__fmul_rn(__fmul_rn(__int2float_rn((int)S[z]), sdv), hs);
                    } else {
                        v = ldexp((double)S[z], -__float_as_int(hs)) * (double)sdv;
                    }
                    ye[(int64_t)entry * d + i] = v;
                }
            }
        }
        tc_fence_before();
    }
    tc_teardown(pp, ALLOC, status);
}

bool tc_grouped_supported(int d, int f) { return d % kTcKT == 0 && f % kTcKT == 0; }

template <int NL>
cudaError_t launch_grouped_tc(const tern_moe_layer *L, int T, const FfnWs &w, cudaStream_t s, int phase) {
    const int d = (int)L->d, f = (int)L->f, E = L->E, k = L->k;
    const int umax = (E < T * k) ? E : T * k;
    int *st = status_word();
    if (phase == 0) {
        const size_t sm = (size_t)kTcStages * (2 * kTcABytes + kTcBBytes);
        cudaFuncSetAttribute(gateup_tc_kernel<NL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        gateup_tc_kernel<NL><<<dim3(umax, (f + kTcM - 1) / kTcM), kTcThreads, sm, s>>>(
            L->gate, L->up, L->gate_scale, L->up_scale, d, f, k, w.n_unique, w.uexp, w.uoff, w.ent,
            (const uint32_t *)w.xw, (const float *)w.xsc, w.h, w.acc_g, w.acc_u, st);
    } else {
        const dim3 grid(umax, (d + kTcDownRB * kTcM - 1) / (kTcDownRB * kTcM));
        if (f <= kTcBWholeMax) {
            const size_t sm = (size_t)kTcStages * kTcABytes + (size_t)kTcBRows * f;
            cudaFuncSetAttribute(down_tc_kernel<NL, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            down_tc_kernel<NL, true><<<grid, kTcThreads, sm, s>>>(
                L->down, L->down_scale, d, f, w.n_unique, w.uexp, w.uoff, w.ent, (const uint32_t *)w.hw,
                (const float *)w.hsc, w.ye, w.acc_d, st);
            return cudaGetLastError();
        }
        const size_t sm = (size_t)kTcStages * (kTcABytes + kTcBBytes);
        cudaFuncSetAttribute(down_tc_kernel<NL, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        down_tc_kernel<NL, false><<<grid, kTcThreads, sm, s>>>(
            L->down, L->down_scale, d, f, w.n_unique, w.uexp, w.uoff, w.ent, (const uint32_t *)w.hw,
            (const float *)w.hsc, w.ye, w.acc_d, st);
    }
    return cudaGetLastError();
}

template cudaError_t launch_grouped_tc<1>(const tern_moe_layer *, int, const FfnWs &, cudaStream_t, int);
template cudaError_t launch_grouped_tc<3>(const tern_moe_layer *, int, const FfnWs &, cudaStream_t, int);

}  // namespace tern
