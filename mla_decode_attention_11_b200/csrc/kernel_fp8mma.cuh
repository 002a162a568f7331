// kernel_fp8mma.cuh -- MLA decode over an FP8 (E4M3) latent cache with the
// codes as tensor-core operands: tcgen05.mma kind::f8f6f4, transposed
// orientation (kv rows on the 128 TMEM lanes, G query rows as N).
//
// The cache format and the definition are those of mla_decode_run_fp8
// (kv_value = kv_scale * e4m3(code)).  Instead of widening every code to f16
// in shared memory, this kernel feeds the staged codes to the MMAs as they
// came from TMA, and brings the other operand to E4M3 instead:
//
//   Q: each query row is scaled by a power of two 2^e (so its largest
//      magnitude is <= 448) and written as the sum of three E4M3 terms
//      t1 + t2 + t3 (t1 = e4m3(x), t2 = e4m3(x - t1), t3 = e4m3(x - t1 - t2)),
//      about 12 significant bits.  The three terms are the N columns
//      [0, G), [G, 2G), [2G, 3G) of one S^T MMA, so every K tile is read
//      once:  S^T[kv, j] = (sum_k S^T_k[kv, j]) * 2^-e_j.
//   P: scaled by 2^4 and written as the sum of two E4M3 terms (about 8
//      significant bits, the precision of the bf16 P of the other kernels);
//      the two terms are the N columns [0, G) and [G, 2G) of the PV MMAs,
//      O^T = O^T_1 + O^T_2.  The reference max is raised only when a column's
//      max exceeds it by more than 4 (base 2), so 2^4 p <= 256 stays inside
//      E4M3 while weights down to 2^-10 of the reference keep normal codes
//      (at scale 1 the smaller ones would fall into the subnormal range and
//      lose precision; a threshold of 1 with 2^7 p rescaled O far more often).
//
// K and V are exact; the errors are the truncation of q (<= 2^-12 relative)
// and of p (<= 2^-8 relative), and fp32 accumulation.  A host-side emulation
// of these splits on N(0, 1) and N(0, 9) data gives out rel-L2 ~1.7e-3 and lse
// errors below 1e-5 against the fp64 oracle.  Everything else --
// the split-KV schedule, the lazy base-2 softmax, sinks, the partials and
// the combine -- is the transposed kernel's.
//
// Warp roles (192 threads):
//   warps 0-3  Q split (once per piece), softmax + epilogue (thread = TMEM lane)
//   warp 4     TMA producer (one elected lane) with an L2 prefetch cursor
//   warp 5     TMEM allocator + MMA issuer (one elected lane)
//
// Shared memory (1024-byte aligned, 64-byte swizzle for the code tiles):
//   pair ring  NP x 16 KB: [128 kv x 128 codes] = value columns 128b .. 128b+127,
//              as two [128 x 64] chunks 8 KB apart
//   rope ring  NR x 8 KB: the [128 kv x 64] rope chunk (columns 512..575)
//   Q terms    9 x [3G x 64] codes, K-major, 64-byte swizzle
//   P terms    [128 kv x 2G] codes, MN-major, 32/64-byte swizzle
//   q scales   G floats (2^-e_j)
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "kernel_transposed.cuh"
#include "ptx.cuh"
#include "schedule.cuh"

namespace mla {

template <int G>
struct Fp8MmaCfg {
    static_assert(G == 16 || G == 32, "query rows per CTA");
    static constexpr int kThreads = 192;
    static constexpr int kQTerms = 3;
    static constexpr int kPTerms = 2;
    static constexpr int NS = kQTerms * G;  // S^T columns
    static constexpr int NO = kPTerms * G;  // O^T columns per 128-row value block
    static constexpr int NP = (G == 16) ? 10 : 8;  // pair slots (a tile needs 4)
    static constexpr int NR = 3;                   // rope slots
    static constexpr int kChunkBytes = kTileKV * kChunk;  // 8 KB: [128 kv x 64 codes]
    static constexpr int kPairBytes = 2 * kChunkBytes;    // 16 KB
    static constexpr int kQChunkBytes = NS * kChunk;      // [3G rows x 64 codes]
    static constexpr int kPBytes = kTileKV * NO;          // [128 kv x 2G codes]
    static constexpr int OFF_PAIR = 0;
    static constexpr int OFF_ROPE = OFF_PAIR + NP * kPairBytes;
    static constexpr int OFF_Q = OFF_ROPE + NR * kChunkBytes;
    static constexpr int OFF_P = OFF_Q + kNumChunks * kQChunkBytes;  // two P buffers (tiles alternate)
    static constexpr int OFF_QS = OFF_P + 2 * kPBytes;             // G floats
    static constexpr int OFF_RED = OFF_QS + G * 4;                 // floats: [2][4][G] max, [4][G] sums
    static constexpr int kRedFloats = 12 * G;
    static constexpr int OFF_BAR = OFF_RED + kRedFloats * 4;
    // barriers: q_ready, q_empty, s_full[2], p_full[2], pv_tile[2], pv_done, drain, group_sync,
    //           pair_full[NP], pair_empty[NP], rope_full[NR], rope_empty[NR]
    static constexpr int kNumBars = 11 + 2 * NP + 2 * NR;
    static constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
    static constexpr int kSmemBytes = OFF_MISC + 64 + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(OFF_Q % 1024 == 0 && OFF_P % 1024 == 0, "swizzled regions start on 1024-byte boundaries");
    // TMEM: O^T blocks at columns [0, 4 NO), then two S^T buffers (tiles alternate)
    static constexpr int kCols = 4 * NO + 2 * NS;
    static constexpr uint32_t kTmemCols = kCols <= 256 ? 256 : 512;
    static constexpr uint32_t kColS = 4 * NO;
    // P^T rows are 2G codes = 32 or 64 bytes
    static constexpr ptx::Swizzle kPSwz = (G == 16) ? ptx::Swizzle::B32 : ptx::Swizzle::B64;
    static constexpr uint32_t kPAtom = 8 * NO;  // 8 rows
    // kind::f8f6f4 with E4M3 A and B: format codes 0, the same bit layout as f16
    static constexpr uint32_t kIdescS = ptx::make_idesc_f16(128, NS, 0, 0);
    static constexpr uint32_t kIdescPV = ptx::make_idesc_f16(128, NO, 1, 1);
    static constexpr float kLazy = 4.f;      // rescale threshold (base-2 units): p <= 16
    static constexpr float kPScaleLog2 = 4.f;  // P is carried as 2^4 p <= 256
    static constexpr float kPScaleInv = 1.f / 16.f;
};

// D[tmem] (+)= A[smem] . B[smem], both E4M3, K = 32 per instruction.
__device__ __forceinline__ void mma_e4m3_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Two floats -> two E4M3 codes (round to nearest even, saturating at +-448);
// the low byte holds `lo`.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// The two values of an E4M3 code pair, exactly.
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t codes) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(codes & 0xFFFFu), __NV_E4M3);
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// The largest e with amax * 2^e <= 448 (0 for amax = 0), kept in [-120, 120].
__device__ __forceinline__ int q_row_exponent(float amax) {
    if (!(amax > 0.f)) return 0;
    int e;
    frexpf(448.f / amax, &e);  // 448 / amax = m 2^e with m in [0.5, 1)
    e -= 1;
    while (e > -120 && ldexpf(amax, e) > 448.f) --e;
    while (e < 120 && ldexpf(amax, e + 1) <= 448.f) ++e;
    return e < -120 ? -120 : (e > 120 ? 120 : e);
}


template <int G>
__global__ void __launch_bounds__(192, 1)
    mla_decode_fp8mma_kernel(const __grid_constant__ CUtensorMap tm_kv, const MainArgs args) {
    using C = Fp8MmaCfg<G>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    uint8_t* pair_smem = smem + C::OFF_PAIR;
    uint8_t* rope_smem = smem + C::OFF_ROPE;
    uint8_t* q_smem = smem + C::OFF_Q;
    uint8_t* p_smem = smem + C::OFF_P;
    float* qscale = reinterpret_cast<float*>(smem + C::OFF_QS);  // per query row: 2^-e * scale_log2
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_ready = bars + 0;     // the softmax threads wrote this piece's Q terms
    uint64_t* q_empty = bars + 1;     // the piece's last S^T MMA completed
    uint64_t* s_full = bars + 2;      // [2] S^T buffer b holds a finished QK^T (tiles alternate)
    uint64_t* p_full = bars + 4;      // [2] P buffer b written by the 128 softmax threads
    uint64_t* pv_tile = bars + 6;     // [2] the PV that read P buffer b has completed
    uint64_t* pv_done = bars + 8;     // the piece's last PV has completed
    uint64_t* drain = bars + 9;
    uint64_t* group_sync = bars + 10; // the 128 softmax threads (bounded, unlike bar.sync)
    uint64_t* pair_full = bars + 11;
    uint64_t* pair_empty = pair_full + C::NP;
    uint64_t* rope_full = pair_empty + C::NP;
    uint64_t* rope_empty = rope_full + C::NR;
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    uint32_t* tmem_base_slot = misc + 0;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    int* b_first_slot = reinterpret_cast<int*>(misc + 2);
    long long* acc_first_slot = reinterpret_cast<long long*>(misc + 4);
    long long* total_slot = reinterpret_cast<long long*>(misc + 6);
    int* split_slot = reinterpret_cast<int*>(misc + 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int p = blockIdx.x / args.NG;  // partition
    const int g = blockIdx.x % args.NG;  // query-row group within the sequence

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        ptx::mbar_init(q_ready, 128);
        ptx::mbar_init(q_empty, 1);
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(s_full + b, 1);
            ptx::mbar_init(p_full + b, 128);
            ptx::mbar_init(pv_tile + b, 1);
        }
        ptx::mbar_init(pv_done, 1);
        ptx::mbar_init(drain, 1);
        ptx::mbar_init(group_sync, 128);
        for (int i = 0; i < C::NP; ++i) {
            ptx::mbar_init(pair_full + i, 1);
            ptx::mbar_init(pair_empty + i, 1);
        }
        for (int i = 0; i < C::NR; ++i) {
            ptx::mbar_init(rope_full + i, 1);
            ptx::mbar_init(rope_empty + i, 1);
        }
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
    }
    if (warp == 5) {
        ptx::tmem_alloc<C::kTmemCols>(tmem_base_slot);
        ptx::tmem_relinquish();
    }
    if (warp == 0) {
        const ScheduleScan sc = schedule_scan_warp(args.seqlens, args.B, args.L_max, args.P, args.split_tiles);
        const long long total = sc.units;
        const long long T = (total + args.P - 1) / args.P;
        int bf;
        long long af;
        locate_warp(args.seqlens, args.B, args.L_max, sc.S, static_cast<long long>(p) * T, &bf, &af);
        if (lane == 0) {
            *b_first_slot = bf;
            *acc_first_slot = af;
            *total_slot = total;
            *split_slot = sc.S;
        }
        if (blockIdx.x == 0)
            for (int b = lane; b < args.B; b += 32) clamp_len(args.seqlens[b], args.L_max, args.status);
    }
    if (warp == 4 && lane == 0) ptx::prefetch_tmap(&tm_kv);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;
    // the split-KV combine (launched after this kernel as a programmatic
    // dependent) may start scheduling its CTAs; it waits for this grid's results
    ptx::launch_dependents();

    PieceWalker walker;
    {
        const long long total = *total_slot;
        const long long T = (total + args.P - 1) / args.P;
        walker.seqlens = args.seqlens;
        walker.B = args.B;
        walker.L_max = args.L_max;
        walker.p = p;
        walker.S = *split_slot;
        walker.k = 0;
        walker.start = static_cast<long long>(p) * T;
        walker.end = walker.start + T < total ? walker.start + T : total;
        walker.b = *b_first_slot;
        walker.acc = *acc_first_slot;
    }
    const uint64_t tmo = args.timeout_ns;

    if (warp == 4) {
        // ============================================================ TMA producer
        if (ptx::elect_one()) {
            uint32_t pair_cnt = 0, rope_cnt = 0;
            int unit = 0;
            bool ok = true;
            // L2 prefetch cursor `prefetch_tiles` tiles ahead of the loads,
            // across piece boundaries (a tile's 9 chunk boxes)
            PieceWalker pf_walker = walker;
            Piece pf_pc{};
            bool pf_live = false, pf_started = false;
            int pf_t = 0;
            auto prefetch_next = [&](bool issue) {
                if (!pf_live) return;
                int r0 = pf_t * kTileKV;
                if (r0 + kTileKV > pf_pc.L) r0 = pf_pc.L - kTileKV;
                if (issue)
                    for (int j = 0; j < kNumChunks; ++j) ptx::tma_prefetch_3d(&tm_kv, j * kChunk, r0, pf_pc.b);
                if (++pf_t == pf_pc.tile_hi) {
                    pf_live = pf_walker.next(pf_pc);
                    if (pf_live) pf_t = pf_pc.tile_lo;
                }
            };
            Piece pc;
            while (ok && walker.next(pc)) {
                for (int t = pc.tile_lo; t < pc.tile_hi && ok; ++t) {
                    if (!pf_started) {
                        pf_started = true;
                        pf_live = args.prefetch_tiles > 0 && pf_walker.next(pf_pc);
                        pf_t = pf_live ? pf_pc.tile_lo : 0;
                        prefetch_next(false);  // this tile: loaded now
                        for (int i = 1; i < args.prefetch_tiles; ++i) prefetch_next(true);
                    }
                    prefetch_next(true);
                    int row0 = t * kTileKV;
                    if (row0 + kTileKV > pc.L) row0 = pc.L - kTileKV;  // end-aligned last tile
                    {
                        const uint32_t s = rope_cnt % C::NR;
                        ok = ptx::mbar_wait_bounded(rope_empty + s, ((rope_cnt / C::NR) & 1) ^ 1, tmo);
                        if (!ok) break;
                        ptx::mbar_arrive_expect_tx(rope_full + s, C::kChunkBytes);
                        if (!(blockIdx.x == 0 && unit == args.stall_unit))
                            ptx::tma_load_3d(rope_smem + s * C::kChunkBytes, &tm_kv, rope_full + s,
                                             (kNumChunks - 1) * kChunk, row0, pc.b);
                        ++unit;
                        ++rope_cnt;
                    }
                    for (int pp = 0; pp < 4; ++pp) {
                        const uint32_t s = pair_cnt % C::NP;
                        ok = ptx::mbar_wait_bounded(pair_empty + s, ((pair_cnt / C::NP) & 1) ^ 1, tmo);
                        if (!ok) break;
                        ptx::mbar_arrive_expect_tx(pair_full + s, C::kPairBytes);
                        if (!(blockIdx.x == 0 && unit == args.stall_unit)) {
                            uint8_t* dst = pair_smem + s * C::kPairBytes;
                            ptx::tma_load_3d(dst, &tm_kv, pair_full + s, (2 * pp) * kChunk, row0, pc.b);
                            ptx::tma_load_3d(dst + C::kChunkBytes, &tm_kv, pair_full + s, (2 * pp + 1) * kChunk,
                                             row0, pc.b);
                        }
                        ++unit;
                        ++pair_cnt;
                    }
                }
            }
            if (!ok) {
                atomicOr(args.status, kStatusTimeout);
                *abort_flag = 1;
            }
            // drain: every load this thread armed must land before the CTA exits (bounded)
            for (uint32_t i = 0; i < C::NP && i < pair_cnt; ++i) {
                const uint32_t use = pair_cnt - 1 - i;
                ptx::mbar_wait_bounded(pair_full + (use % C::NP), (use / C::NP) & 1, tmo);
            }
            for (uint32_t i = 0; i < C::NR && i < rope_cnt; ++i) {
                const uint32_t use = rope_cnt - 1 - i;
                ptx::mbar_wait_bounded(rope_full + (use % C::NR), (use / C::NR) & 1, tmo);
            }
        }
        __syncwarp();
    } else if (warp == 5) {

        // ============================================================ MMA issuer
        // Within a piece, QK^T of tile t+1 goes to the tensor pipe before the
        // issuer waits for tile t's softmax, so the pipe works on the next S^T
        // while the softmax runs; S^T and P are double-buffered by tile parity.
        // Pipe order per piece: S(0), S(1), PV(0), S(2), PV(1), ..., PV(last):
        // S(t+2) follows PV(t), so when the softmax sees S(t+2) complete, PV(t)
        // has stopped reading P buffer t % 2 and S^T buffer t % 2 is free again.
        // Not across pieces: the next piece's Q terms are written by the softmax
        // threads after this piece's epilogue, which waits for the last PV.
        if (ptx::elect_one()) {
            uint32_t pair_cnt = 0, rope_cnt = 0, piece_cnt = 0, tile_cnt = 0;
            bool ok = true;
            const uint32_t q_base = ptx::smem_u32(q_smem);
            const uint32_t p_base0 = ptx::smem_u32(p_smem);
            uint32_t slots[2][4];  // the pair slots of the tiles in flight, by tile parity
            // S^T(t) = K . [Q1 Q2 Q3]^T for global tile index u (rope chunk first, then the 8 value chunks)
            auto issue_qk = [&](uint32_t u, bool last) -> bool {
                const uint32_t sb = u & 1;
                const uint32_t tm_S = tmem_base + C::kColS + sb * C::NS;
                const uint32_t rs = rope_cnt % C::NR;
                if (!ptx::mbar_wait_bounded(rope_full + rs, (rope_cnt / C::NR) & 1, tmo)) return false;
                ptx::tc_fence_after();
                {
                    const uint32_t a0 = ptx::smem_u32(rope_smem + rs * C::kChunkBytes);
                    const uint32_t b0 = q_base + (kNumChunks - 1) * C::kQChunkBytes;
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {  // 32 codes = 32 bytes per MMA
                        const uint64_t da = ptx::make_smem_desc(a0 + kk * 32, 16, 512, ptx::Swizzle::B64);
                        const uint64_t db = ptx::make_smem_desc(b0 + kk * 32, 16, 512, ptx::Swizzle::B64);
                        mma_e4m3_ss(tm_S, da, db, C::kIdescS, kk > 0 ? 1u : 0u);
                    }
                }
                ptx::mma_commit(rope_empty + rs);
                ++rope_cnt;
                for (int pp = 0; pp < 4; ++pp) {
                    const uint32_t s = (pair_cnt + pp) % C::NP;
                    slots[sb][pp] = s;
                    if (!ptx::mbar_wait_bounded(pair_full + s, ((pair_cnt + pp) / C::NP) & 1, tmo)) return false;
                    ptx::tc_fence_after();
                    const uint32_t pbase = ptx::smem_u32(pair_smem + s * C::kPairBytes);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int c = 2 * pp + h;
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint64_t da = ptx::make_smem_desc(pbase + h * C::kChunkBytes + kk * 32, 16,
                                                                    512, ptx::Swizzle::B64);
                            const uint64_t db = ptx::make_smem_desc(q_base + c * C::kQChunkBytes + kk * 32, 16,
                                                                    512, ptx::Swizzle::B64);
                            mma_e4m3_ss(tm_S, da, db, C::kIdescS, 1u);
                        }
                    }
                }
                pair_cnt += 4;
                if (last) ptx::mma_commit(q_empty);
                ptx::mma_commit(s_full + sb);
                return true;
            };
            Piece pc;
            while (ok && walker.next(pc)) {
                ok = ptx::mbar_wait_bounded(q_ready, piece_cnt & 1, tmo);
                if (!ok) break;
                const int n = pc.tile_hi - pc.tile_lo;
                ok = issue_qk(tile_cnt, n == 1);
                for (int i = 0; ok && i < n; ++i) {
                    const uint32_t u = tile_cnt;
                    if (i + 1 < n) {
                        ok = issue_qk(u + 1, i + 2 == n);
                        if (!ok) break;
                    }
                    // ---------------- O^T += V^T . [P1 P2]^T  (after the softmax wrote tile u's P terms)
                    const uint32_t pb = u & 1;
                    ok = ptx::mbar_wait_bounded(p_full + pb, (u >> 1) & 1, tmo);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const uint32_t p_base = p_base0 + pb * C::kPBytes;
                    for (int pp = 0; pp < 4; ++pp) {
                        const uint32_t vbase = ptx::smem_u32(pair_smem + slots[pb][pp] * C::kPairBytes);
                        const uint32_t tm_O = tmem_base + pp * C::NO;
#pragma unroll
                        for (int kk = 0; kk < kTileKV / 32; ++kk) {
                            // A = V^T block: M = 128 value columns (two 64-wide atoms 8 KB
                            // apart), K = 32 kv rows (four 8-row groups of 64 bytes)
                            const uint64_t da =
                                ptx::make_smem_desc(vbase + kk * 2048, C::kChunkBytes, 512, ptx::Swizzle::B64);
                            // B = the P terms: K = 32 kv rows (four atoms), N = 2G (one atom wide)
                            const uint64_t db = ptx::make_smem_desc(p_base + kk * 4 * C::kPAtom, C::kPBytes,
                                                                    C::kPAtom, C::kPSwz);
                            mma_e4m3_ss(tm_O, da, db, C::kIdescPV, (i > 0 || kk > 0) ? 1u : 0u);
                        }
                        ptx::mma_commit(pair_empty + slots[pb][pp]);
                    }
                    ptx::mma_commit(pv_tile + pb);
                    if (i + 1 == n) ptx::mma_commit(pv_done);
                    ++tile_cnt;
                }
                ++piece_cnt;
            }
            if (!ok) {
                atomicOr(args.status, kStatusTimeout);
                *abort_flag = 1;
            }
            // drain: all MMAs this thread issued must complete before TMEM is freed
            ptx::mma_commit(drain);
            ptx::mbar_wait_bounded(drain, 0, tmo);
        }
        __syncwarp();
    } else {
        // ============================================================ Q split, softmax + epilogue (warps 0-3)
        const int row_in_tile = warp * 32 + lane;  // TMEM lane = kv row (S^T) = value column (O^T)
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
        const int my_col = col_of_lane<G>(lane);
        const bool writes_col = (G == 32) || ((lane & 1) == 0);
        constexpr int kThrPerRow = 128 / G;             // Q split: threads per query row (consecutive lanes)
        const int qj = threadIdx.x / kThrPerRow;        // the query row this thread splits
        const int qpart = threadIdx.x % kThrPerRow;
        constexpr int kUnitsPerTerm = G / 16;           // 16-byte units of one P term in a kv row
        uint32_t tile_cnt = 0, piece_cnt = 0, sync_cnt = 0;
        bool ok = true;
        // bounded barrier over the 128 softmax threads
        auto group_barrier = [&]() -> bool {
            ptx::mbar_arrive(group_sync);
            const bool r = ptx::mbar_wait_bounded(group_sync, sync_cnt & 1, tmo);
            ++sync_cnt;
            return r;
        };
        Piece pc;
        while (ok && walker.next(pc)) {
            // ---------------- this piece's Q rows as three E4M3 terms, each row scaled by 2^e
            if (piece_cnt > 0) {  // the previous piece's S^T MMAs no longer read the terms
                ok = ptx::mbar_wait_bounded(q_empty, (piece_cnt - 1) & 1, tmo);
                if (!ok) break;
            }
            {
                // this thread's 16-byte units qpart, qpart + kThrPerRow, ... of the row,
                // loaded at once (one round trip to memory)
                constexpr int kQUnits = kDqk / 8 / kThrPerRow;
                static_assert(kQUnits * kThrPerRow * 8 == kDqk, "q units per thread");
                const uint4* qrow =
                    reinterpret_cast<const uint4*>(args.q + (static_cast<size_t>(pc.b) * args.R + g * G + qj) * kDqk);
                uint4 qv[kQUnits];
#pragma unroll
                for (int i = 0; i < kQUnits; ++i) qv[i] = __ldg(qrow + qpart + i * kThrPerRow);
                float amax = 0.f;
#pragma unroll
                for (int i = 0; i < kQUnits; ++i) {
                    const uint32_t w[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
                        amax = ptx::fmax3(amax, fabsf(f.x), fabsf(f.y));
                    }
                }
#pragma unroll
                for (int o = kThrPerRow / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                const int e = q_row_exponent(amax);
                if (qpart == 0) qscale[qj] = ldexpf(args.scale_log2, -e);
                const float up = ldexpf(1.f, e);
#pragma unroll
                for (int i = 0; i < kQUnits; ++i) {
                    const int sg = qpart + i * kThrPerRow;
                    const uint32_t w[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
                    float x[8];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
                        x[2 * i] = f.x * up;
                        x[2 * i + 1] = f.y * up;
                    }
                    uint32_t tw[3][2];  // term k: 8 codes in two words
#pragma unroll
                    for (int k = 0; k < 3; ++k) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t c01 = f32x2_to_e4m3x2(x[4 * h], x[4 * h + 1]);
                            const uint32_t c23 = f32x2_to_e4m3x2(x[4 * h + 2], x[4 * h + 3]);
                            tw[k][h] = c01 | (c23 << 16);
                            const float2 v01 = e4m3x2_to_f32x2(c01);
                            const float2 v23 = e4m3x2_to_f32x2(c23);
                            x[4 * h] -= v01.x;
                            x[4 * h + 1] -= v01.y;
                            x[4 * h + 2] -= v23.x;
                            x[4 * h + 3] -= v23.y;
                        }
                    }
                    // columns d0 .. d0+7 of chunk d0 / 64: half of one 16-byte unit of the row
                    const int d0 = sg * 8;
                    const uint32_t u = static_cast<uint32_t>((d0 % kChunk) / 16);
                    const uint32_t half8 = static_cast<uint32_t>((d0 % 16) / 8) * 8;
                    uint8_t* chunk = q_smem + (d0 / kChunk) * C::kQChunkBytes;
#pragma unroll
                    for (int k = 0; k < 3; ++k)
                        *reinterpret_cast<uint2*>(chunk + swz_offset(static_cast<uint32_t>(k * G + qj), u, 64) +
                                                  half8) = make_uint2(tw[k][0], tw[k][1]);
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(q_ready);
            ok = ptx::mbar_wait_bounded(q_ready, piece_cnt & 1, tmo);  // every row's scale is in qscale
            if (!ok) break;

            float m_ref[G];
            float l_part[G];
#pragma unroll
            for (int j = 0; j < G; ++j) {
                m_ref[j] = -INFINITY;
                l_part[j] = 0.f;
            }
            for (int t = pc.tile_lo; t < pc.tile_hi; ++t) {
                const bool first = (t == pc.tile_lo);
                int row0 = t * kTileKV;
                if (row0 + kTileKV > pc.L) row0 = pc.L - kTileKV;
                const int kv_row = row0 + row_in_tile;
                const bool valid = (kv_row >= t * kTileKV) && (kv_row < pc.L);

                const uint32_t sb = tile_cnt & 1;  // S^T and P buffer of this tile
                ok = ptx::mbar_wait_bounded(s_full + sb, (tile_cnt >> 1) & 1, tmo);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t col_s = C::kColS + sb * C::NS;
                float x[G];
#pragma unroll
                for (int c0 = 0; c0 < G; c0 += 16) {
                    uint32_t r[16];
                    float acc[16];
                    ptx::tmem_ld_16(lane_addr + col_s + c0, r);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[j] = __uint_as_float(r[j]);
#pragma unroll
                    for (int k = 1; k < C::kQTerms; ++k) {
                        ptx::tmem_ld_16(lane_addr + col_s + k * G + c0, r);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) acc[j] += __uint_as_float(r[j]);
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) x[c0 + j] = valid ? acc[j] * qscale[c0 + j] : -INFINITY;
                }
                // column max over the tile's 128 kv rows
                float* redmax = red + (tile_cnt & 1) * 4 * G;
                const float wmax = warp_reduce_scatter<G, true>(x, lane);
                if (writes_col) redmax[warp * G + my_col] = wmax;
                ok = group_barrier();
                if (!ok) break;
                float tmax[G];
#pragma unroll
                for (int j = 0; j < G; j += 4) {
                    float4 a = *reinterpret_cast<const float4*>(redmax + 0 * G + j);
                    const float4 b1 = *reinterpret_cast<const float4*>(redmax + 1 * G + j);
                    const float4 b2 = *reinterpret_cast<const float4*>(redmax + 2 * G + j);
                    const float4 b3 = *reinterpret_cast<const float4*>(redmax + 3 * G + j);
                    tmax[j + 0] = fmaxf(fmaxf(a.x, b1.x), fmaxf(b2.x, b3.x));
                    tmax[j + 1] = fmaxf(fmaxf(a.y, b1.y), fmaxf(b2.y, b3.y));
                    tmax[j + 2] = fmaxf(fmaxf(a.z, b1.z), fmaxf(b2.z, b3.z));
                    tmax[j + 3] = fmaxf(fmaxf(a.w, b1.w), fmaxf(b2.w, b3.w));
                }
                // lazy rescale (threshold kLazy, so 2^4 p <= 256 < 448), uniform branch
                bool grow = false;
#pragma unroll
                for (int j = 0; j < G; ++j) grow |= (tmax[j] > m_ref[j] + C::kLazy);
                if (first) {
#pragma unroll
                    for (int j = 0; j < G; ++j) m_ref[j] = tmax[j];
                } else if (grow) {
                    // O^T must hold the previous tile's PV before it is rescaled (this
                    // tile's PV waits for the P written below)
                    ok = ptx::mbar_wait_bounded(pv_tile + ((tile_cnt - 1) & 1), ((tile_cnt - 1) >> 1) & 1, tmo);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    float alpha[G];
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        const float mn = fmaxf(m_ref[j], tmax[j]);
                        alpha[j] = ex2_approx(m_ref[j] - mn);
                        m_ref[j] = mn;
                        l_part[j] *= alpha[j];
                    }
                    // O^T columns of query j (both P terms) *= alpha[j]
#pragma unroll
                    for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
                        for (int c0 = 0; c0 < C::NO; c0 += 16) {
                            uint32_t r[16];
                            ptx::tmem_ld_16(lane_addr + blk * C::NO + c0, r);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha[(c0 % G) + j]);
                            ptx::tmem_st_16(lane_addr + blk * C::NO + c0, r);
                        }
                    }
                    ptx::tmem_wait_st();
                }
                // P terms of this kv row: 2^4 p = t1 + t2 (E4M3), t1 in bytes [0, G), t2 in [G, 2G);
                // P buffer sb was last read by the PV of tile - 2, which the tensor pipe ran
                // before this tile's S^T
                uint8_t* p_buf = p_smem + sb * C::kPBytes;
                uint32_t w1[G / 4], w2[G / 4];
#pragma unroll
                for (int j = 0; j < G; j += 2) {
                    const float p0 = ex2_approx(x[j] - m_ref[j] + C::kPScaleLog2);
                    const float p1 = ex2_approx(x[j + 1] - m_ref[j + 1] + C::kPScaleLog2);
                    const uint32_t t1 = f32x2_to_e4m3x2(p0, p1);
                    const float2 v1 = e4m3x2_to_f32x2(t1);
                    const uint32_t t2 = f32x2_to_e4m3x2(p0 - v1.x, p1 - v1.y);
                    const float2 v2 = e4m3x2_to_f32x2(t2);
                    l_part[j] += v1.x + v2.x;  // the weights the MMAs use
                    l_part[j + 1] += v1.y + v2.y;
                    if ((j & 2) == 0) {
                        w1[j / 4] = t1;
                        w2[j / 4] = t2;
                    } else {
                        w1[j / 4] |= t1 << 16;
                        w2[j / 4] |= t2 << 16;
                    }
                }
#pragma unroll
                for (int u = 0; u < kUnitsPerTerm; ++u) {
                    *reinterpret_cast<uint4*>(p_buf + swz_offset(row_in_tile, u, C::NO)) =
                        make_uint4(w1[4 * u], w1[4 * u + 1], w1[4 * u + 2], w1[4 * u + 3]);
                    *reinterpret_cast<uint4*>(p_buf + swz_offset(row_in_tile, kUnitsPerTerm + u, C::NO)) =
                        make_uint4(w2[4 * u], w2[4 * u + 1], w2[4 * u + 2], w2[4 * u + 3]);
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                ptx::mbar_arrive(p_full + sb);
                ++tile_cnt;
            }
            if (!ok) break;
            // ---------------- epilogue: (O1 + O2) / l -> out (or a partial), lse
            ok = ptx::mbar_wait_bounded(pv_done, piece_cnt & 1, tmo);
            if (!ok) break;
            ptx::tc_fence_after();
            float* redsum = red + 8 * G;
            {
                const float ws = warp_reduce_scatter<G, false>(l_part, lane);
                if (writes_col) redsum[warp * G + my_col] = ws;
            }
            ok = group_barrier();
            if (!ok) break;
            const bool sink_here = (args.sinks != nullptr) && (pc.slot < 0);
            float* fin = red + (tile_cnt & 1) * 4 * G;
            if (row_in_tile < G) {
                const int j = row_in_tile;
                const int qr = g * G + j;  // query row within the sequence
                float mj = 0.f;
#pragma unroll
                for (int jj = 0; jj < G; ++jj)
                    if (jj == j) mj = m_ref[jj];
                // the sums and O carry the 2^4 of P: l is unscaled here, O in fin
                float lj = (redsum[0 * G + j] + redsum[1 * G + j] + redsum[2 * G + j] + redsum[3 * G + j]) *
                           C::kPScaleInv;
                float c = 1.f;
                if (sink_here) c = fold_sink(mj, lj, args.sinks[qr % args.H] * kLog2e);
                fin[j] = c / lj * args.o_scale * C::kPScaleInv;
                const float lse_nat = (mj + log2f(lj)) * 0.69314718055994530942f;
                if (pc.slot < 0)
                    args.lse[static_cast<size_t>(pc.b) * args.R + qr] = lse_nat;
                else
                    args.part_lse[static_cast<size_t>(pc.slot) * args.R + qr] = lse_nat;
            }
            ok = group_barrier();
            if (!ok) break;
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
                const int dv = blk * 128 + row_in_tile;
#pragma unroll
                for (int c0 = 0; c0 < G; c0 += 16) {
                    uint32_t r1[16], r2[16];
                    ptx::tmem_ld_16(lane_addr + blk * C::NO + c0, r1);
                    ptx::tmem_ld_16(lane_addr + blk * C::NO + G + c0, r2);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float o = (__uint_as_float(r1[j]) + __uint_as_float(r2[j])) * fin[c0 + j];
                        const int qr = g * G + c0 + j;
                        if (pc.slot < 0)
                            args.out[(static_cast<size_t>(pc.b) * args.R + qr) * kDv + dv] = __float2bfloat16_rn(o);
                        else
                            args.part_o[(static_cast<size_t>(pc.slot) * args.R + qr) * kDv + dv] = o;
                    }
                }
            }
            ptx::tc_fence_before();
            // the next piece reuses the sums buffer only after everyone read it
            ok = group_barrier();
            ++piece_cnt;
        }
        if (!ok) {
            atomicOr(args.status, kStatusTimeout);
            *abort_flag = 1;
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc<C::kTmemCols>(tmem_base);
    }
}

}  // namespace mla
