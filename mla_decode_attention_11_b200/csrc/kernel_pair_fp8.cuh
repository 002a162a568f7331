// kernel_pair_fp8.cuh -- MLA decode over an FP8 (E4M3) latent cache for
// 128-row query groups, on a CTA pair (cluster of 2, tcgen05 cta_group::2 with
// kind::f8f6f4).
//
// The dataflow, warp roles, pipelines, schedule, softmax and epilogue are those
// of mla_decode_pair_kernel (kernel_pair.cuh); what changes is the operand
// format.  The staged E4M3 codes of the cache are the B operands as TMA wrote
// them (64-byte swizzle: K for S in 64-code chunks, K-major; V for PV in
// 64-column chunks, MN-major), and the A operands are brought to E4M3:
//
//   Q: each query row is scaled by a power of two 2^e (its largest magnitude
//      <= 448) and written as two E4M3 terms t1 = e4m3(x), t2 = e4m3(x - t1),
//      about 8 significant bits (the precision of a bf16 q).  Both terms
//      multiply the same K chunk into the same S accumulator, so
//      S = (t1 + t2) K^T and the softmax multiplies each row by 2^-e.
//   P: carried as 2^4 p, rounded to f16 and written as two E4M3 terms
//      t1 = e4m3(h), t2 = e4m3(h - t1) (about 8 significant bits, the
//      precision of the bf16 P of the other kernels); both multiply the same
//      V chunk into O.  The row sum adds the fp32 weights 2^4 p, so the
//      factor 2^4 cancels in O / l; the reference max is raised only when a
//      row max exceeds it by more than 4 (base 2), so 2^4 p <= 256 stays
//      inside E4M3 while weights down to 2^-10 of the reference keep normal
//      codes.  (A threshold of 1 with 2^7 p rescaled O several times per
//      row, each time waiting for the PV in flight.)
//
// With K = 32 codes per instruction and two terms, the MMA count and the
// tensor time per tile are those of the bf16 pair kernel; the cache bytes
// loaded per tile (and the TMA bytes) are half.  The Q terms are written by
// the softmax warps at the start of each piece (plain loads of the bf16 q);
// the leader's QK^T issuer waits until both CTAs have written theirs.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "kernel_fp8mma.cuh"
#include "kernel_transposed.cuh"
#include "ptx.cuh"
#include "schedule.cuh"

namespace mla {

// An f16 pair -> two E4M3 codes (round to nearest even, saturating at +-448);
// the low byte holds the low half.
__device__ __forceinline__ uint32_t f16x2_to_e4m3x2(__half2 h) {
    return static_cast<uint32_t>(
        __nv_cvt_halfraw2_to_fp8x2(*reinterpret_cast<const __half2_raw*>(&h), __NV_SATFINITE, __NV_E4M3));
}

// The two values of an E4M3 code pair as an f16 pair, exactly.
__device__ __forceinline__ __half2 e4m3x2_to_f16x2(uint32_t codes) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(codes & 0xFFFFu), __NV_E4M3);
    return *reinterpret_cast<const __half2*>(&h);
}

template <int NK, int NV, int NS, int NP>
struct PairFp8Cfg {
    static constexpr int kThreads = 256;
    static constexpr int kRows = 64;                          // query rows per CTA
    static constexpr int kQTerms = 2;
    static constexpr int kQChunk = kRows * kChunk;            // 4 KB: one term of [64 rows x 64 codes]
    static constexpr int kKChunk = 64 * kChunk;               // 4 KB: [64 own kv rows x 64 codes]
    static constexpr int kVChunk = kTileKV * kChunk;          // 8 KB: [128 kv x 64 value codes]
    static constexpr int kVSlot = 2 * kVChunk;                // 16 KB: this CTA's 128 of one N = 256 half
    static constexpr int kPChunk = kRows * 64;                // 4 KB: one term of [64 rows x 64 keys]
    static constexpr int kPTerm = 2 * kPChunk;                // 8 KB: one term of a tile's 128 keys
    static constexpr int OFF_Q = 0;                           // [term][chunk] 4 KB each: 72 KB
    static constexpr int OFF_K = OFF_Q + kQTerms * kNumChunks * kQChunk;
    static constexpr int OFF_V = OFF_K + NK * kKChunk;
    static constexpr int OFF_P = OFF_V + NV * kVSlot;
    static constexpr int kPBuf = 2 * kPTerm;                  // one P tile: [term][64-key half] 4 KB each
    static_assert(NP == 1 || NP == 2, "one or two P buffers (they double as the epilogue's store stages)");
    static constexpr int kStagesPerWarp = NP * kPBuf / (4 * 4096);  // 4 KB epilogue stages per softmax warp
    static_assert(kStagesPerWarp >= 1, "epilogue stages");
    static constexpr int OFF_RED = OFF_P + NP * kPBuf;         // floats: [2][128] max, [128] sum, [128] q amax, [64] q scale
    static constexpr int OFF_BAR = OFF_RED + 576 * 4;
    // q_full, q_empty, pv_done[NP], drain_s, drain_pv, group_sync, s_full[NS], p_full[NS], p_local[NS],
    // k_full[NK], k_empty[NK], v_full[NV], v_empty[NV]
    static constexpr int kNumBars = 6 + NP + 3 * NS + 2 * NK + 2 * NV;
    static constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
    static constexpr int kSmemBytes = OFF_MISC + 64;
    static constexpr uint32_t kTmemCols = 512;                 // O: [0,256), S buffers from 256, 64 each
    static constexpr uint32_t kColS = 256;
    static_assert(NS >= 2 && 256 + 64 * NS <= 512, "S buffers must fit next to O in TMEM");
    static_assert(NS <= 4, "one 4-byte forwarding slot per S buffer in the 64-byte misc area (words 12..15)");
    // kind::f8f6f4 with E4M3 A and B: format codes 0 (the bit layout of the f16 descriptor)
    static constexpr uint32_t kIdescS = ptx::make_idesc_f16(128, 128, 0, 0);
    static constexpr uint32_t kIdescPV = ptx::make_idesc_f16(128, 256, 0, 1);
    static constexpr float kLazy = 4.f;        // rescale threshold (base 2): 2^4 p <= 256
    static constexpr float kPScaleLog2 = 4.f;  // P carried as 2^4 p
    static constexpr float kPScaleInv = 1.f / 16.f;
    static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && OFF_P % 1024 == 0, "swizzle atoms");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// D[tmem of both CTAs] (+)= A . B with the CTA pair, both operands E4M3
// codes, K = 32 per instruction; issued by one thread of the leader CTA.
__device__ __forceinline__ void mma_e4m3_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int NK, int NV, int NS, int NP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(256, 1)
    mla_decode_pair_fp8_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                               const __grid_constant__ CUtensorMap tm_pf, const __grid_constant__ CUtensorMap tm_out,
                               const __grid_constant__ CUtensorMap tm_part, const MainArgs args) {
    using C = PairFp8Cfg<NK, NV, NS, NP>;
    extern __shared__ __align__(1024) uint8_t smem[];

    uint8_t* q_smem = smem + C::OFF_Q;
    uint8_t* k_smem = smem + C::OFF_K;
    uint8_t* v_smem = smem + C::OFF_V;
    uint8_t* p_smem = smem + C::OFF_P;
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars + 0;            // leader: both CTAs' softmax threads wrote the piece's Q terms
    uint64_t* q_empty = bars + 1;           // the piece's last QK^T has completed (multicast)
    uint64_t* pv_done = bars + 2;           // [NP] the PV that read P buffer b has completed
    uint64_t* drain_s = pv_done + NP;
    uint64_t* drain_pv = drain_s + 1;
    uint64_t* group_sync = drain_pv + 1;
    uint64_t* s_full = group_sync + 1;      // [NS] S buffer b holds a finished QK^T
    uint64_t* p_full = s_full + NS;         // [NS] leader: the tile in S buffer b is through both softmaxes
                                            //      (its S read, its P written in both CTAs): 128 arrivals
                                            //      and 4 transaction bytes stored by the follower
    uint64_t* p_local = p_full + NS;        // [NS] follower: the same, for this CTA's 128 softmax threads
    uint64_t* k_full = p_local + NS;
    uint64_t* k_empty = k_full + NK;
    uint64_t* v_full = k_empty + NK;
    uint64_t* v_empty = v_full + NV;
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    uint32_t* tmem_base_slot = misc + 0;
    int* b_first_slot = reinterpret_cast<int*>(misc + 2);
    long long* acc_first_slot = reinterpret_cast<long long*>(misc + 4);
    long long* total_slot = reinterpret_cast<long long*>(misc + 6);
    int* split_slot = reinterpret_cast<int*>(misc + 8);  // schedule chunk size of this run (0: balanced)
    uint32_t* fwd_slot = misc + 12;                       // [NS] leader: target of the follower's P-ready store

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();  // 0 = leader (issues the pair MMAs)
    const bool leader = (rank == 0);
    const int pair_id = blockIdx.x >> 1;
    const int p = pair_id / args.NG;  // partition
    const int g = pair_id % args.NG;  // 128-row query group within the sequence
    const uint64_t tmo = args.timeout_ns;
    // the shared-memory carve-up assumes a 1024-byte aligned base (128-byte swizzle atoms)
    const bool smem_ok = (ptx::smem_u32(smem) & 1023u) == 0;

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        ptx::mbar_init(q_full, 256);  // 128 softmax threads of each CTA
        ptx::mbar_init(q_empty, 1);
        for (int i = 0; i < NS; ++i) {
            ptx::mbar_init(s_full + i, 1);
            ptx::mbar_init(p_full + i, 128);   // leader's 128 softmax threads (+ 4 tx bytes from the follower)
            ptx::mbar_init(p_local + i, 128);  // follower's 128 softmax threads
        }
        for (int i = 0; i < NP; ++i) ptx::mbar_init(pv_done + i, 1);
        ptx::mbar_init(drain_s, 1);
        ptx::mbar_init(drain_pv, 1);
        ptx::mbar_init(group_sync, 128);
        for (int i = 0; i < NK; ++i) {
            ptx::mbar_init(k_full + i, 1);
            ptx::mbar_init(k_empty + i, 1);
        }
        for (int i = 0; i < NV; ++i) {
            ptx::mbar_init(v_full + i, 1);
            ptx::mbar_init(v_empty + i, 1);
        }
        ptx::fence_mbarrier_init();
        if (!smem_ok) atomicOr(args.status, kStatusTimeout);
    }
    if (warp == 6) {
        ptx::tmem_alloc_pair<C::kTmemCols>(tmem_base_slot);
        ptx::tmem_relinquish_pair();
    }
    if (warp == 0) {
        const ScheduleScan sc = schedule_scan_warp(args.seqlens, args.B, args.L_max, args.P, args.split_tiles);
        const int S_eff = sc.S;
        const long long total = sc.units;
        const long long T = (total + args.P - 1) / args.P;
        int bf;
        long long af;
        locate_warp(args.seqlens, args.B, args.L_max, S_eff, static_cast<long long>(p) * T, &bf, &af);
        if (lane == 0) {
            *b_first_slot = bf;
            *acc_first_slot = af;
            *total_slot = total;
            *split_slot = S_eff;
        }
        if (blockIdx.x == 0)
            for (int b = lane; b < args.B; b += 32) clamp_len(args.seqlens[b], args.L_max, args.status);
    }
    if (warp == 4 && lane == 0) {
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_pf);
        ptx::prefetch_tmap(&tm_out);
        ptx::prefetch_tmap(&tm_part);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync_all();  // peer barriers initialised before any cross-CTA signal
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
        walker.b = smem_ok ? *b_first_slot : args.B;  // misaligned smem: do nothing
        walker.acc = *acc_first_slot;
    }
    // shared::cluster address of the leader's Q barrier
    const uint32_t lead_q_full = ptx::mapa_shared(ptx::smem_u32(q_full), 0);
    const bool stall_cta = (blockIdx.x == 0);

    if (warp == 4) {
        // ============================================================ Q + K producer
        if (ptx::elect_one()) {
            // K as one 64-code chunk of this CTA's 64 kv rows per slot; the L2
            // prefetch of a tile as one box of 64 rows x all 9 chunks
            uint32_t k_cnt = 0, piece_cnt = 0;
            int unit = 0;
            bool ok = true;
            // L2 prefetch cursor, `prefetch_tiles` tiles ahead of the K loads
            // through this partition's tiles, across piece boundaries.  A tile
            // is prefetched whole (this CTA's 64 rows, K and V columns alike).
            // The cursor skips the first tile (loaded at once), so nothing
            // queues ahead of the loads the first MMA needs.
            PieceWalker pf_walker = walker;
            Piece pf_pc{};
            bool pf_live = false, pf_started = false;
            int pf_t = 0;
            auto prefetch_next = [&](bool issue) {
                if (!pf_live) return;
                int row0 = pf_t * kTileKV;
                if (row0 + kTileKV > pf_pc.L) row0 = pf_pc.L - kTileKV;
                if (issue) ptx::tma_prefetch_4d(&tm_pf, 0, row0 + static_cast<int>(rank) * 64, 0, pf_pc.b);
                if (++pf_t == pf_pc.tile_hi) {
                    pf_live = pf_walker.next(pf_pc);
                    if (pf_live) pf_t = pf_pc.tile_lo;
                }
            };
            Piece pc;
            while (ok && walker.next(pc)) {
                ++unit;  // (a piece's Q is written by the softmax warps; the unit numbering matches the bf16 kernel)
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
                    if (row0 + kTileKV > pc.L) row0 = pc.L - kTileKV;
                    const int krow = row0 + static_cast<int>(rank) * 64;
                    for (int jj = 0; jj < kNumChunks; ++jj) {
                        const int j = (jj == 0) ? 8 : jj - 1;  // rope chunk first
                        const uint32_t s = k_cnt % NK;
                        ok = ptx::mbar_wait_bounded(k_empty + s, ((k_cnt / NK) & 1) ^ 1, tmo);
                        if (!ok) break;
                        if (leader) ptx::mbar_arrive_expect_tx(k_full + s, 2 * C::kKChunk);
                        if (!(stall_cta && unit == args.stall_unit))
                            ptx::tma_load_3d_pair(k_smem + s * C::kKChunk, &tm_k,
                                                  ptx::mapa_shared(ptx::smem_u32(k_full + s), 0), j * kChunk,
                                                  krow, pc.b);  // x: j * 64 codes = 64 j bytes
                        ++unit;
                        ++k_cnt;
                    }
                }
                ++piece_cnt;
            }
            if (!ok) atomicOr(args.status, kStatusTimeout);
            // before teardown, every load this CTA pair may still have in flight
            // must have landed: the leader counts both CTAs' bytes, so it waits
            // (bounded) for the last phase it armed on each K slot
            // (a drain that runs out means a load never landed: recorded as a timeout)
            if (leader) {
                bool drained = true;
                const uint32_t n_k = k_cnt < static_cast<uint32_t>(NK) ? k_cnt : static_cast<uint32_t>(NK);
                for (uint32_t i = 0; i < n_k; ++i) {
                    const uint32_t c = k_cnt - 1 - i;
                    drained &= ptx::mbar_wait_bounded(k_full + c % NK, (c / NK) & 1, tmo);
                }
                if (!drained) atomicOr(args.status, kStatusTimeout);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ============================================================ V producer
        if (ptx::elect_one()) {
            uint32_t v_cnt = 0;
            bool ok = true;
            Piece pc;
            while (ok && walker.next(pc)) {
                for (int t = pc.tile_lo; t < pc.tile_hi && ok; ++t) {
                    int row0 = t * kTileKV;
                    if (row0 + kTileKV > pc.L) row0 = pc.L - kTileKV;
                    for (int i = 0; i < 2; ++i) {
                        const uint32_t s = v_cnt % NV;
                        ok = ptx::mbar_wait_bounded(v_empty + s, ((v_cnt / NV) & 1) ^ 1, tmo);
                        if (!ok) break;
                        if (leader) ptx::mbar_arrive_expect_tx(v_full + s, 2 * C::kVSlot);
                        // this CTA's value columns [col0, col0 + 128): two adjacent chunks, one box
                        const int col0 = 256 * i + 128 * static_cast<int>(rank);
                        ptx::tma_load_4d_pair(v_smem + s * C::kVSlot, &tm_v,
                                              ptx::mapa_shared(ptx::smem_u32(v_full + s), 0), 0, row0, col0 / kChunk,
                                              pc.b);
                        ++v_cnt;
                    }
                }
            }
            if (!ok) atomicOr(args.status, kStatusTimeout);
            if (leader) {  // as for K: the last armed phase of each V slot has landed
                bool drained = true;
                const uint32_t n_v = v_cnt < static_cast<uint32_t>(NV) ? v_cnt : static_cast<uint32_t>(NV);
                for (uint32_t i = 0; i < n_v; ++i) {
                    const uint32_t c = v_cnt - 1 - i;
                    drained &= ptx::mbar_wait_bounded(v_full + c % NV, (c / NV) & 1, tmo);
                }
                if (!drained) atomicOr(args.status, kStatusTimeout);
            }
        }
        __syncwarp();
    } else if (warp == 6) {
        // ============================================================ QK^T issuer (leader only)
        if (leader && ptx::elect_one()) {
            bool ok = true;
            constexpr uint16_t kBoth = 0x3;
            // descriptors of the chunk / slot bases (64-byte rows, 64-byte swizzle,
            // 8-row atoms 512 bytes apart); an MMA adds (byte offset >> 4)
            const uint64_t dq0 = ptx::make_smem_desc(ptx::smem_u32(q_smem), 16, 512, ptx::Swizzle::B64);
            const uint64_t dk0 = ptx::make_smem_desc(ptx::smem_u32(k_smem), 16, 512, ptx::Swizzle::B64);
            uint32_t ks = 0, kph = 0;        // K ring slot and phase
            uint32_t sb = 0, sph = 0;        // S buffer and its use parity
            uint32_t u = 0, piece_cnt = 0;   // global tile index, piece count
            Piece pc;
            while (ok && walker.next(pc)) {
                // both CTAs' Q terms are written (the follower's arrivals are cluster-scope releases)
                ok = ptx::mbar_wait_bounded_cluster(q_full, piece_cnt & 1, tmo);
                for (int t = pc.tile_lo; ok && t < pc.tile_hi; ++t) {
                    // S buffer sb was last filled by tile u - NS: both softmaxes must be done with it
                    if (u >= static_cast<uint32_t>(NS)) {
                        ok = ptx::mbar_wait_bounded_cluster(p_full + sb, sph ^ 1, tmo);
                        if (!ok) break;
                    }
                    const uint32_t tm_S = tmem_base + C::kColS + 64 * sb;
                    for (int jj = 0; jj < kNumChunks; ++jj) {
                        const uint32_t j = (jj == 0) ? 8u : static_cast<uint32_t>(jj - 1);  // rope chunk first
                        ok = ptx::mbar_wait_bounded(k_full + ks, kph, tmo);
                        if (!ok) break;
                        ptx::tc_fence_after();
                        const uint64_t db = dk0 + ((ks * C::kKChunk) >> 4);
                        // both Q terms against the same K chunk, 32 codes per MMA
#pragma unroll
                        for (int tq = 0; tq < C::kQTerms; ++tq) {
                            const uint64_t da = dq0 + (((tq * kNumChunks + j) * C::kQChunk) >> 4);
#pragma unroll
                            for (int kk = 0; kk < 2; ++kk)
                                mma_e4m3_ss_pair(tm_S, da + 2 * kk, db + 2 * kk, C::kIdescS, (jj | tq | kk) ? 1u : 0u);
                        }
                        ptx::mma_commit_pair_mc(k_empty + ks, kBoth);
                        if (++ks == NK) {
                            ks = 0;
                            kph ^= 1;
                        }
                    }
                    if (!ok) break;
                    if (t == pc.tile_hi - 1) ptx::mma_commit_pair_mc(q_empty, kBoth);
                    ptx::mma_commit_pair_mc(s_full + sb, kBoth);
                    if (++sb == NS) {
                        sb = 0;
                        sph ^= 1;
                    }
                    ++u;
                }
                ++piece_cnt;
            }
            if (!ok) atomicOr(args.status, kStatusTimeout);
            // drain: every MMA this thread issued must complete before TMEM is freed
            ptx::mma_commit_pair_mc(drain_s, 0x1);
            ptx::mbar_wait_bounded(drain_s, 0, tmo);
        }
        __syncwarp();
    } else if (warp == 7 && !leader) {
        // ============================================================ P-ready forwarder (follower)
        // One cluster-scope release per tile (the st.async's complete-tx), made here
        // instead of by every softmax thread.
        if (ptx::elect_one()) {
            bool ok = true;
            uint32_t u = 0;
            Piece pc;
            while (ok && walker.next(pc)) {
                for (int t = pc.tile_lo; ok && t < pc.tile_hi; ++t, ++u) {
                    const uint32_t b = u % NS;
                    ok = ptx::mbar_wait_bounded(p_local + b, (u / NS) & 1, tmo);
                    // a 4-byte st.async into the leader's fwd slot, counted on its p_full
                    if (ok)
                        ptx::st_async_u32(ptx::mapa_shared(ptx::smem_u32(fwd_slot + b), 0), u,
                                          ptx::mapa_shared(ptx::smem_u32(p_full + b), 0));
                }
            }
            if (!ok) atomicOr(args.status, kStatusTimeout);
        }
        __syncwarp();
    } else if (warp == 7) {
        // ============================================================ PV issuer (leader only)
        if (leader && ptx::elect_one()) {
            bool ok = true;
            constexpr uint16_t kBoth = 0x3;
            // P terms: K-major, 64-byte rows (64 keys); V: MN-major, two 64-column
            // chunks kVChunk apart (LBO), 8-key atoms of 512 bytes (SBO)
            const uint64_t dp0 = ptx::make_smem_desc(ptx::smem_u32(p_smem), 16, 512, ptx::Swizzle::B64);
            const uint64_t dv0 = ptx::make_smem_desc(ptx::smem_u32(v_smem), C::kVChunk, 512, ptx::Swizzle::B64);
            uint32_t vs = 0, vph = 0;  // V ring slot and phase
            uint32_t u = 0;            // global tile index
            Piece pc;
            while (ok && walker.next(pc)) {
                for (int t = pc.tile_lo; ok && t < pc.tile_hi; ++t) {
                    const bool first = (t == pc.tile_lo);  // O starts over for a new piece
                    const uint32_t pb = (NP == 2) ? (u & 1) : 0;
                    ok = ptx::mbar_wait_bounded_cluster(p_full + (u % NS), (u / NS) & 1, tmo);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const uint64_t dpb = dp0 + ((pb * C::kPBuf) >> 4);
                    for (int i = 0; i < 2; ++i) {
                        ok = ptx::mbar_wait_bounded(v_full + vs, vph, tmo);
                        if (!ok) break;
                        ptx::tc_fence_after();
                        const uint64_t db = dv0 + ((vs * C::kVSlot) >> 4);
                        // 32 keys per MMA (4 steps), both P terms against the same V rows
#pragma unroll
                        for (int kk = 0; kk < kTileKV / 32; ++kk) {
#pragma unroll
                            for (int tp = 0; tp < 2; ++tp) {
                                const uint64_t da =
                                    dpb + ((tp * C::kPTerm + (kk >> 1) * C::kPChunk + (kk & 1) * 32) >> 4);
                                mma_e4m3_ss_pair(tmem_base + 128 * i, da, db + ((kk * 2048) >> 4), C::kIdescPV,
                                                 (first && kk == 0 && tp == 0) ? 0u : 1u);
                            }
                        }
                        ptx::mma_commit_pair_mc(v_empty + vs, kBoth);
                        if (++vs == NV) {
                            vs = 0;
                            vph ^= 1;
                        }
                    }
                    if (!ok) break;
                    ptx::mma_commit_pair_mc(pv_done + pb, kBoth);
                    ++u;
                }
            }
            if (!ok) atomicOr(args.status, kStatusTimeout);
            ptx::mma_commit_pair_mc(drain_pv, 0x1);
            ptx::mbar_wait_bounded(drain_pv, 0, tmo);
        }
        __syncwarp();
    } else {
        // ============================================================ softmax + epilogue (warps 0-3)
        const int L_id = warp * 32 + lane;  // TMEM lane
        const int r = L_id & 63;            // query row within this CTA's 64
        const int h = L_id >> 6;            // which 64 keys of the tile (S), which 128 dv of each N=256 (O)
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
        uint32_t tile_cnt = 0, sync_cnt = 0, piece_cnt = 0;
        bool ok = true;
        // scores are scaled by cs before exp2; a non-positive scale is applied to
        // the raw scores up front (cs = 1 after that), so that the row max of the
        // raw scores times cs is the scaled row max
        float* qamax = red + 384;  // [128] this thread's |q| max, for the row's other thread
        float* qscale = red + 512; // [64] 2^-e of each row
        auto group_barrier = [&]() -> bool {
            ptx::mbar_arrive(group_sync);
            const bool rr = ptx::mbar_wait_bounded(group_sync, sync_cnt & 1, tmo);
            ++sync_cnt;
            return rr;
        };
        Piece pc;
        while (ok && walker.next(pc)) {
            // ---------------- the piece's Q as two E4M3 terms.  Thread (r, h) takes
            // 16-byte units [36h, 36h + 36) of row r in three batches of 12, each
            // batch's loads issued together: the row max over the three, then the
            // terms (the last batch still in registers, the first two reloaded),
            // written after the previous piece's last QK^T has read the old ones
            {
                if (piece_cnt > 0) {
                    ok = ptx::mbar_wait_bounded(q_empty, (piece_cnt - 1) & 1, tmo);
                    if (!ok) break;
                }
                constexpr int kQUnits = kDqk / 8 / 2;  // 16-byte units (8 bf16) per thread
                constexpr int kQBatch = 12;
                constexpr int kQBatches = kQUnits / kQBatch;
                static_assert(kQBatches * kQBatch == kQUnits, "q batches");
                const uint4* qsrc = reinterpret_cast<const uint4*>(
                    args.q + (static_cast<size_t>(pc.b) * args.R + g * 128 + static_cast<int>(rank) * 64 + r) * kDqk) +
                    kQUnits * h;
                uint4 qv[kQBatch];
                float amax = 0.f;
#pragma unroll
                for (int bt = 0; bt < kQBatches; ++bt) {
#pragma unroll
                    for (int i = 0; i < kQBatch; ++i) qv[i] = __ldg(qsrc + bt * kQBatch + i);
#pragma unroll
                    for (int i = 0; i < kQBatch; ++i) {
                        const uint32_t w[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
                            amax = ptx::fmax3(amax, fabsf(f.x), fabsf(f.y));
                        }
                    }
                }
                qamax[L_id] = amax;
                ok = group_barrier();
                if (!ok) break;
                amax = fmaxf(amax, qamax[L_id ^ 64]);
                const int e = q_row_exponent(amax);
                if (h == 0) qscale[r] = ldexpf(1.f, -e);
                const float up = ldexpf(1.f, e);
#pragma unroll 1
                for (int bt = kQBatches - 1; bt >= 0; --bt) {
                    if (bt != kQBatches - 1) {
#pragma unroll
                        for (int i = 0; i < kQBatch; ++i) qv[i] = __ldg(qsrc + bt * kQBatch + i);
                    }
#pragma unroll
                    for (int i = 0; i < kQBatch; ++i) {
                        const uint32_t w[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
                        float x[8];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
                            x[2 * j] = f.x * up;
                            x[2 * j + 1] = f.y * up;
                        }
                        uint32_t tw[2][2];  // term k: 8 codes in two words
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                const uint32_t c01 = f32x2_to_e4m3x2(x[4 * hh], x[4 * hh + 1]);
                                const uint32_t c23 = f32x2_to_e4m3x2(x[4 * hh + 2], x[4 * hh + 3]);
                                tw[k][hh] = c01 | (c23 << 16);
                                const float2 v01 = e4m3x2_to_f32x2(c01);
                                const float2 v23 = e4m3x2_to_f32x2(c23);
                                x[4 * hh] -= v01.x;
                                x[4 * hh + 1] -= v01.y;
                                x[4 * hh + 2] -= v23.x;
                                x[4 * hh + 3] -= v23.y;
                            }
                        }
                        // codes d0 .. d0+7 of chunk d0 / 64: half of one 16-byte unit of row r
                        const int d0 = (kQUnits * h + bt * kQBatch + i) * 8;
                        const uint32_t u = static_cast<uint32_t>((d0 % kChunk) / 16);
                        const uint32_t half8 = static_cast<uint32_t>((d0 % 16) / 8) * 8;
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            uint8_t* chunk = q_smem + (k * kNumChunks + d0 / kChunk) * C::kQChunk;
                            *reinterpret_cast<uint2*>(chunk + swz_offset(static_cast<uint32_t>(r), u, 64) + half8) =
                                make_uint2(tw[k][0], tw[k][1]);
                        }
                    }
                }
                ptx::fence_proxy_async_smem();
                ok = group_barrier();  // every row's scale is in qscale
                if (!ok) break;
                // the leader's QK^T issuer waits for both CTAs' terms
                if (leader) ptx::mbar_arrive(q_full);
                else ptx::mbar_arrive_cluster(lead_q_full);
                ++piece_cnt;
            }
            const float row_cs = args.scale_log2 * qscale[r];  // score scale of this row (base 2)
            float m_ref = -INFINITY;  // reference max (base 2) of the row, the same in both of its threads
            float l_part = 0.f;       // this thread's share of the row sum (of 2^4 p), relative to m_ref
            for (int t = pc.tile_lo; t < pc.tile_hi; ++t) {
                const bool first = (t == pc.tile_lo);
                int row0 = t * kTileKV;
                if (row0 + kTileKV > pc.L) row0 = pc.L - kTileKV;
                const int kv0 = row0 + 64 * h;       // key of column j is kv0 + j
                const int lo = t * kTileKV;          // keys below lo belong to the previous tile
                const uint32_t buf = tile_cnt % NS;
                ok = ptx::mbar_wait_bounded(s_full + buf, (tile_cnt / NS) & 1, tmo);
                if (!ok) break;
                ptx::tc_fence_after();
                float x[64];
                {
                    uint32_t ra[32], rb[32];
                    ptx::tmem_ld_32(lane_addr + C::kColS + 64 * buf, ra);
                    ptx::tmem_ld_32(lane_addr + C::kColS + 64 * buf + 32, rb);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        x[j] = __uint_as_float(ra[j]);
                        x[32 + j] = __uint_as_float(rb[j]);
                    }
                }
                float cs = row_cs;
                if (!(cs > 0.f)) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) x[j] *= cs;
                    cs = 1.f;
                }
                // only the end-aligned last tile of a sequence holds keys of the
                // previous tile (below lo); every key of a tile is below L
                if (row0 < lo) {
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        if (kv0 + j < lo) x[j] = -INFINITY;
                }
                // this thread's max (a tree of three-input maxima), then published
                // for the row's other thread; the exchange completes while the
                // exps below run
                const float mloc = ptx::max64(x) * cs;
                float* redmax = red + (tile_cnt & 1) * 128;
                redmax[L_id] = mloc;
                ptx::mbar_arrive(group_sync);
                // 2^4 P[r][64h .. 64h+63] = exp2(x * cs - m_ref + 4) as two E4M3
                // terms.  Past a piece's first tile the reference max is known
                // before this tile's max, so P is computed at once; it is redone
                // only when the row max outgrew the reference by more than 4
                // (2^4 p <= 256).
                uint32_t packed[2][16];  // term k: 64 codes in 16 words
                float lsum = 0.f;
                auto exps = [&](float m) {
                    // the exponents and the row sum two lanes at a time (packed fp32)
                    float2 ls = make_float2(0.f, 0.f);
                    const float mm = m - C::kPScaleLog2;
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float a[4];
#pragma unroll
                        for (int i = 0; i < 4; i += 2) {
                            const float2 tt = ptx::ffma2(make_float2(x[4 * e + i], x[4 * e + i + 1]),
                                                         make_float2(cs, cs), make_float2(-mm, -mm));
                            a[i] = ex2_approx(tt.x);
                            a[i + 1] = ex2_approx(tt.y);
                        }
                        // Two terms through f16 pairs: h = a rounded to f16 (relative
                        // error 2^-11); first term = h rounded to E4M3; the remainder
                        // h - first is exact in f16 (a multiple of h's spacing, at most
                        // half the first term's spacing, so under 8 significant bits);
                        // second term = the remainder rounded to E4M3.  The pair holds a
                        // to about 2^-8 relative (below E4M3's normal range, to its
                        // subnormal spacing 2^-9: under 2^-13 of the row sum, which
                        // holds a term of 2^4).  The row sum takes the fp32 weights,
                        // as in the bf16 kernel.
                        const __half2 h01 = __floats2half2_rn(a[0], a[1]);
                        const __half2 h23 = __floats2half2_rn(a[2], a[3]);
                        const uint32_t c01 = f16x2_to_e4m3x2(h01);
                        const uint32_t c23 = f16x2_to_e4m3x2(h23);
                        const uint32_t d01 = f16x2_to_e4m3x2(__hsub2(h01, e4m3x2_to_f16x2(c01)));
                        const uint32_t d23 = f16x2_to_e4m3x2(__hsub2(h23, e4m3x2_to_f16x2(c23)));
                        ls = ptx::fadd2(ls, ptx::fadd2(make_float2(a[0], a[1]), make_float2(a[2], a[3])));
                        packed[0][e] = c01 | (c23 << 16);
                        packed[1][e] = d01 | (d23 << 16);
                    }
                    lsum = ls.x + ls.y;
                };
                if (!first) exps(m_ref);
                ok = ptx::mbar_wait_bounded(group_sync, sync_cnt & 1, tmo);
                ++sync_cnt;
                if (!ok) break;
                const float mrow = fmaxf(mloc, redmax[L_id ^ 64]);
                float alpha = 1.f;
                bool grow = false;
                if (first) {
                    m_ref = mrow;
                    exps(m_ref);
                } else if (mrow > m_ref + C::kLazy) {
                    grow = true;
                    alpha = ex2_approx(m_ref - mrow);
                    m_ref = mrow;
                    l_part *= alpha;
                    exps(m_ref);
                }
                l_part += lsum;
                const bool warp_grow = __any_sync(0xffffffffu, grow);
                const uint32_t pb = (NP == 2) ? (tile_cnt & 1) : 0;
                // the P buffer is free once the PV that last read it completed
                // (NP = 1: the previous tile's; NP = 2: the one two tiles back)
                if (NP == 1 ? !first : (t >= pc.tile_lo + 2)) {
                    const uint32_t v = tile_cnt - NP;
                    ok = ptx::mbar_wait_bounded(pv_done + pb, (NP == 2) ? ((v >> 1) & 1) : (v & 1), tmo);
                    if (!ok) break;
                }
                if (warp_grow) {
                    // O must hold every earlier tile before it is rescaled
                    if (NP == 2) {
                        const uint32_t v = tile_cnt - 1;
                        ok = ptx::mbar_wait_bounded(pv_done + (v & 1), (v >> 1) & 1, tmo);
                        if (!ok) break;
                    }
                    ptx::tc_fence_after();
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
#pragma unroll
                        for (int c0 = 0; c0 < 128; c0 += 32) {
                            uint32_t rr[32];
                            ptx::tmem_ld_32(lane_addr + 128 * i + c0, rr);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 32; ++j) rr[j] = __float_as_uint(__uint_as_float(rr[j]) * alpha);
                            ptx::tmem_st_32(lane_addr + 128 * i + c0, rr);
                        }
                    }
                    ptx::tmem_wait_st();
                }
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    uint8_t* pchunk = p_smem + pb * C::kPBuf + k * C::kPTerm + h * C::kPChunk;
#pragma unroll
                    for (int uu = 0; uu < 4; ++uu)
                        *reinterpret_cast<uint4*>(pchunk + swz_offset(static_cast<uint32_t>(r), uu, 64)) =
                            make_uint4(packed[k][4 * uu + 0], packed[k][4 * uu + 1], packed[k][4 * uu + 2],
                                       packed[k][4 * uu + 3]);
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                // CTA-scope arrive: the leader's own barrier, or the follower's local one
                // (the leader's thread 0 also arms the 4 bytes the follower's forwarder stores)
                if (leader && L_id == 0) ptx::mbar_arrive_expect_tx(p_full + buf, 4);
                else ptx::mbar_arrive(leader ? (p_full + buf) : (p_local + buf));
                ++tile_cnt;
            }
            if (!ok) break;
            // ---------------- epilogue: O / l -> out (or a partial), lse
            {
                const uint32_t v = tile_cnt - 1;  // the piece's last tile
                ok = (NP == 2) ? ptx::mbar_wait_bounded(pv_done + (v & 1), (v >> 1) & 1, tmo)
                               : ptx::mbar_wait_bounded(pv_done, v & 1, tmo);
            }
            if (!ok) break;
            ptx::tc_fence_after();
            float* redsum = red + 256;
            redsum[L_id] = l_part;
            ok = group_barrier();
            if (!ok) break;
            const int qrow = g * 128 + static_cast<int>(rank) * 64 + r;  // row within the sequence
            // l and O both carry the factor 2^4 of the P terms
            float l_row = (l_part + redsum[L_id ^ 64]) * C::kPScaleInv;
            // a sink applies once per row: to whole sequences here, to cut ones in the combine
            float o_fac = 1.f;
            if (args.sinks != nullptr && pc.slot < 0)
                o_fac = fold_sink(m_ref, l_row, args.sinks[qrow % args.H] * kLog2e);
            const float inv_l = o_fac * args.o_scale * C::kPScaleInv / l_row;
            if (h == 0) {
                const float lse_nat = (m_ref + log2f(l_row)) * 0.69314718055994530942f;
                if (pc.slot < 0)
                    args.lse[static_cast<size_t>(pc.b) * args.R + qrow] = lse_nat;
                else
                    args.part_lse[static_cast<size_t>(pc.slot) * args.R + qrow] = lse_nat;
            }
            // O / l leaves TMEM one 128-byte column block at a time: this warp's
            // 32 rows x 128 bytes are written into a 4 KB stage in the 128-byte
            // swizzle a TMA store expects (lane = row, so each instruction
            // spreads over all banks), and one lane stores the box with TMA.
            // Each warp owns NP 4 KB stages of the P buffers, used in turn:
            // every PV of the piece has completed, and the next piece's P is
            // written only after the closing group barrier.
            {
                constexpr int NST = C::kStagesPerWarp;
                uint8_t* stage = p_smem + warp * (NST * 4096);
                const bool partial = (pc.slot >= 0);
                const int y0 = (partial ? pc.slot : pc.b) * args.R + g * 128 + static_cast<int>(rank) * 64 +
                               32 * (warp & 1);  // first of this warp's 32 rows
                const int nblk = partial ? 8 : 4;  // fp32: 32 columns per box; bf16: 64
#pragma unroll 1
                for (int blk = 0; blk < nblk; ++blk) {
                    const int i = partial ? (blk >> 2) : (blk >> 1);
                    const int c0 = partial ? (blk & 3) * 32 : (blk & 1) * 64;
                    uint32_t ra[32], rb[32];
                    ptx::tmem_ld_32(lane_addr + 128 * i + c0, ra);
                    if (!partial) ptx::tmem_ld_32(lane_addr + 128 * i + c0 + 32, rb);
                    ptx::tmem_wait_ld();
                    if (blk >= NST) {  // the store that last read this stage must be done with it
                        if (lane == 0) ptx::bulk_wait_group_read<NST - 1>();
                        __syncwarp();
                    }
                    uint8_t* sb = stage + (blk % NST) * 4096 + lane * 128;
                    if (partial) {
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            *reinterpret_cast<float4*>(sb + ((k ^ (lane & 7)) << 4)) =
                                make_float4(__uint_as_float(ra[4 * k + 0]) * inv_l, __uint_as_float(ra[4 * k + 1]) * inv_l,
                                            __uint_as_float(ra[4 * k + 2]) * inv_l, __uint_as_float(ra[4 * k + 3]) * inv_l);
                    } else {
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const uint32_t* src = (k < 4) ? (ra + 8 * k) : (rb + 8 * (k - 4));
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const __nv_bfloat162 bv = __floats2bfloat162_rn(__uint_as_float(src[2 * e]) * inv_l,
                                                                                __uint_as_float(src[2 * e + 1]) * inv_l);
                                w[e] = *reinterpret_cast<const uint32_t*>(&bv);
                            }
                            *reinterpret_cast<uint4*>(sb + ((k ^ (lane & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        const int col = 256 * i + 128 * h + c0;  // first value column of the box
                        ptx::tma_store_2d(partial ? &tm_part : &tm_out, stage + (blk % NST) * 4096, col, y0);
                        ptx::bulk_commit_group();
                    }
                }
                if (lane == 0) ptx::bulk_wait_group_read<0>();  // stages free for the next piece's P
                __syncwarp();
            }
            ptx::tc_fence_before();
            ok = group_barrier();  // sums buffer and P buffers reused by the next piece
        }
        if (!ok) atomicOr(args.status, kStatusTimeout);
        // the output stores must be complete before this CTA's shared memory goes away
        if (lane == 0) ptx::bulk_wait_group<0>();
        __syncwarp();
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync_all();  // both CTAs finished (the leader drained its MMAs) before freeing TMEM
    if (warp == 6) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair<C::kTmemCols>(tmem_base);
    }
}

}  // namespace mla
