// gemm.cu -- block-scaled MX GEMM on the 5th-generation tensor cores (sm_100a).
//
//   Y[M, N] = bf16( sum_k deqA[m, k] * deqW[n, k] + bias[n] )
//
// with A the quantized activation and W the MXFP4 weight, both K-major with one
// E8M0 scale per 32 elements along K.  This is the native W4A4 / W4A8 linear of the
// blog "Quark Mixed-Precision Quantization for Wan2.2 Video Generation on AMD
// Instinct GPUs" (section "Quantization formats", "Kernel note"): W4A4 runs
// tcgen05.mma kind::mxf4 (both operands E2M1, K = 64 per instruction); W4A8 runs
// kind::mxf8f6f4 with A in E4M3 and the E2M1 weight expanded by TMA into the
// byte-padded shared-memory form (K = 32 per instruction).
//
// Structure (one CTA per SM, persistent over output tiles).  Two variants: a lone
// CTA owning 128 x 256 tiles, and a CTA pair (a 2-CTA cluster on one TPC, MMAs with
// cta_group::2) owning 256 x 256 tiles, where each CTA loads its own 128 activation
// rows and half of the 256 weight rows, so each SM moves 2/3 of the bytes per FLOP.
//   warp 0      TMA producer (each CTA): A / W tiles (128-byte swizzle) and the
//               scale-factor atoms (512-byte chunks, as 2-D TMA boxes) into the
//               shared-memory ring; a pair's loads all complete on the leader's barrier;
//   warp 1      MMA issuer (leader CTA): issues the block-scaled MMAs of each landed
//               stage into the TMEM accumulators; its commits release the stage (in
//               both CTAs) and the stage's TMEM scale buffer; in every CTA this warp
//               allocates and frees TMEM;
//   warps 2..5  epilogue (each CTA): tcgen05.ld 32 columns at a time, + bias, -> bf16,
//               staged in swizzled shared memory and written with TMA stores;
//   warp 6      scale copies (leader CTA): copies each stage's scale atoms into one of
//               kSfBufs TMEM scale buffers (tcgen05.cp 32x128b.warpx4) ahead of the
//               MMAs.  tcgen05 operations of one thread run in order, so copies issued
//               by the MMA thread would stall behind its MMAs; from their own thread
//               they overlap them.
// The same kernel runs bf16 x bf16 stages (kind::f16): the SVDQuant low-rank branch's
// stages ahead of the block-scaled ones, or every stage of a plain bf16 GEMM.  One lone-CTA
// bf16 variant (kQA) adds warps 7..14, which MX-quantize each landed stage of A from
// shared memory and release it beside the MMAs (the branch's u and x's codes from one
// read of x).
// L2 policies: the weight is loaded evict-last (it is reused by every m-block and fits
// in L2), the output is stored evict-first.
// TMEM (512 columns): accumulator slot 0 = [0, 256), slot 1 = [kAccCol1, kAccCol1 + 256),
// kSfBufs scale buffers above.  The two slots share 256 - kAccCol1 columns; the
// epilogue drains those first and signals it, so the next tile's MMAs can start while
// the rest of the previous accumulator is still being written out.  (The kQA variant,
// whose output is at most 128 columns and which uses no scale buffers, puts slot 1 at
// [256, 512) and shares nothing.)
// Every wait is bounded; a wait that runs out records MXQ_ERR_TIMEOUT in a device
// status word and the kernel winds down (in-flight copies and MMAs drained, TMEM
// freed) instead of hanging.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <type_traits>

#include "mx_elem.cuh"
#include "mxq_internal.h"
#include "ptx.cuh"

namespace mxq {

__device__ uint32_t g_device_status;

namespace {

constexpr int BN = 256;                   // output columns per tile (both variants): 256 or 192
// Warp roles: 0 TMA producer, 1 MMA issuer, then the epilogue warps, then one scale-copy
// warp.  The bf16 epilogue has four warps, one per TMEM lane quarter; the quantizing
// epilogue eight, two per lane quarter taking alternate chunks, so that its GELU
// arithmetic has twice the warps to hide latency with.
template <int kOut>
constexpr int kEpiWarpsOf = kOut ? 8 : 4;
template <int kOut>
constexpr int kThreadsOf = 64 + 32 * kEpiWarpsOf<kOut> + 32;
// A bf16 GEMM that also MX-quantizes its A operand (the bf16 activation) as its stages
// stream through shared memory: eight more warps, one MX block of an A row per thread.
constexpr int kQaWarps = 8;
template <int kOut, bool kQA>
constexpr int kThreadsFor = kThreadsOf<kOut> + (kQA ? 32 * kQaWarps : 0);
constexpr uint32_t kEpiBuf = 32 * 64;     // 32 rows x 32 bf16
constexpr uint32_t kTmemCols = 512;
// TMEM columns: accumulator slot 0 [0, BN), slot 1 [kAccCol1, kAccCol1 + BN) (sharing
// BN - kAccCol1 columns with slot 0 when they do not both fit), then kSfBufs
// scale-factor buffers of 24 columns: SFA at +0 (4 columns per k-atom), SFB at +8
// (8 columns per k-atom: the 256 weight rows of the 128-aligned window holding the tile).
constexpr uint32_t kSfBufs = 3;            // scale buffers in TMEM (the copy thread runs ahead)
constexpr uint32_t kSfBufCols = 24;
constexpr uint32_t kSfCol = kTmemCols - kSfBufs * kSfBufCols;
// slot 1 follows slot 0 when there is room, otherwise the two slots share columns
constexpr uint32_t kAccCol1 = kSfCol - BN < uint32_t(BN) ? kSfCol - BN : uint32_t(BN);
constexpr int kOverlapChunks = kAccCol1 < uint32_t(BN) ? (BN - kAccCol1 + 31) / 32 : 0;  // shared 32-col chunks
static_assert(BN == 256 || BN == 192, "tile width");
static_assert(kAccCol1 + BN <= kSfCol, "TMEM plan");
constexpr uint64_t kWaitNs = 1000000000ull;
// Epilogue chunk registers in flight (32 columns each): three, so the shared columns
// (kOverlapChunks chunks) leave TMEM after one wait.
constexpr int kLdBufs = 3;
static_assert(kOverlapChunks <= kLdBufs, "the shared columns must fit the first round of loads");
static_assert(BN / 32 >= 3, "the quantizing epilogue's ring holds three chunks");
// The kernel that quantizes its A (kQA) writes at most 128 output columns and copies no
// scales into TMEM, so its two accumulator slots take [0, 256) and [256, 512) and share
// nothing; its epilogue drains the four chunks that can hold output, two loads in flight
// (which keeps it inside the registers the kernel's 480 threads leave each thread).
template <bool kQA>
constexpr uint32_t kAcc1Of = kQA ? 256u : kAccCol1;
template <bool kQA>
constexpr int kOverlapOf = kQA ? 0 : kOverlapChunks;
template <bool kQA>
constexpr int kLdBufsOf = kQA ? 2 : kLdBufs;
template <bool kQA>
constexpr int kChunksOf = kQA ? 4 : BN / 32;

// Output of the epilogue: bf16 y = acc + bias; or the next layer's MX-quantized input,
// h = bf16(GELU(bf16(acc + bias))) -- or h = bf16(acc + bias) when the launch asks for no
// activation (Params::gelu) -- as E2M1 / E4M3 codes with tiled E8M0 scales (and h itself
// in bf16 when asked for).
constexpr int kOutBf16 = 0;
constexpr int kOutGeluE2M1 = 1;
constexpr int kOutGeluE4M3 = 2;
// The same two quantizing epilogues for launches that ask for no h: without the bf16
// staging buffers they have room for the bf16 variant's six pipeline stages, and h's store
// path is compiled out (1-2 % faster than the variants with h, paired A/B at 720p).
constexpr int kOutQE2M1 = 3;
constexpr int kOutQE4M3 = 4;
template <int kOut>
constexpr bool kOutE4M3 = kOut == kOutGeluE4M3 || kOut == kOutQE4M3;
template <int kOut>
constexpr bool kOutEbuf = kOut <= kOutGeluE4M3;  // bf16 staging buffers (y, or h on request)

// Shared-memory plan of one CTA.  kPair = 1: the CTA owns a 128 x 256 tile and loads
// all 256 weight rows; kPair = 2: a CTA pair owns a 256 x 256 tile, each CTA loads its
// own 128 activation rows and 128 of the 256 weight rows (the pair MMA reads both).
// kQA (the bf16 GEMM that quantizes its A, output at most 128 wide): B stages of 128 rows
// and no scale stages, which leaves room for six stages of the activation in flight.
template <int kPair, int kOut, bool kQA = false>
struct Cfg {
    // the quantizing epilogue's code staging takes one pipeline stage's worth of memory,
    // unless the launch writes no h (no bf16 staging then)
    static constexpr int kStages = kQA ? 6 : kPair == 2 ? ((kOut && kOutEbuf<kOut>) ? 5 : 6) : (kOut ? 3 : 4);
    static constexpr int BM = 128 * kPair;
    static constexpr int kRowsB = kQA ? 128 : BN / kPair;
    static constexpr uint32_t kStageA = 128 * 128;
    static constexpr uint32_t kStageB = kRowsB * 128;
    static constexpr uint32_t kStageSFA = kQA ? 0 : 2 * 512;       // up to two k-atoms
    static constexpr uint32_t kStageSFB = kQA ? 0 : 2 * 2 * 512;   // both 128-row halves of the tile
    static constexpr uint32_t kOffA = 0;
    static constexpr uint32_t kOffB = kOffA + kStages * kStageA;
    static constexpr uint32_t kOffSFA = kOffB + kStages * kStageB;
    static constexpr uint32_t kOffSFB = kOffSFA + kStages * kStageSFA;
    static constexpr uint32_t kOffEpi = kOffSFB + kStages * kStageSFB;
    static constexpr uint32_t kQBuf = kOutE4M3<kOut> ? 32 * 32 : 32 * 16;  // 32 rows of one block's codes
    // code staging buffers per warp: two, or one for E4M3, whose larger codes would
    // otherwise leave no room for the GELU table
    static constexpr int kQBufs = kOutE4M3<kOut> ? 1 : 2;
    static constexpr int kEpiWarps = kEpiWarpsOf<kOut>;
    static constexpr uint32_t kOffQ = kOffEpi + (kOutEbuf<kOut> ? kEpiWarps * 2 * kEpiBuf : 0u);
    static constexpr uint32_t kOffLut = kOffQ + (kOut ? kEpiWarps * kQBufs * kQBuf : 0u);  // GELU table
    static constexpr uint32_t kOffBar = kOffLut + (kOut ? kGeluTableBytes : 0u);
    static constexpr uint32_t kNumBars = 2 * kStages + 6 + 2 * kSfBufs;
    static constexpr uint32_t kSmemBytes = kOffBar + kNumBars * 8 + 16;
    static constexpr int kGroupM = 32;  // tile rows (tiles along M) per rasterization group
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kOffB % 1024 == 0 && kOffSFA % 1024 == 0 && kOffEpi % 1024 == 0, "alignment");
};

struct Params {
    const __nv_bfloat16* bias;
    int M, N, K;
    int m_blocks, n_blocks, num_tiles, k_stages;
    uint32_t debug;
    // quantizing epilogue: tiled scales of the output (K = N), their k-atoms, rows padded
    // to 128, and whether h is also written in bf16 through map_y
    uint8_t* q_sf;
    uint32_t q_atoms_k;
    int q_rows_pad;
    int write_h;
    int gelu;     // quantizing epilogue: 1 = h is GELU of the linear's output, 0 = h is that output
    float alpha;  // per-tensor activation scale applied to the sums (1 for MX activations)
    // low-rank branch: stages of 64 K-elements of u (activation, bf16 [M, r]) and B^T
    // (bf16 [N, r]) MMA'd (kind::f16) into the accumulator before the block-scaled stages
    int lr_stages;
    int mma_n;  // N of the bf16 MMAs: BN, or the output width rounded up to 16 for a lone CTA's only tile column
    // A quantized on the side (kQA): codes [M, K/2] (E2M1) or [M, K] (E4M3) and tiled scales
    uint8_t* qa_codes;
    uint8_t* qa_sf;
    uint32_t qa_atoms_k;
    int qa_fmt;
};

__device__ __forceinline__ void record_status(uint32_t code) { atomicCAS(&g_device_status, 0u, code); }

template <int kGroupM>
__device__ __forceinline__ void tile_coords(int t, int m_blocks, int n_blocks, int& mb, int& nb)
{
    const int per_group = kGroupM * n_blocks;
    const int gid = t / per_group;
    const int first_m = gid * kGroupM;
    const int gsize = min(kGroupM, m_blocks - first_m);
    const int local = t - gid * per_group;
    nb = local / gsize;
    mb = first_m + (local - nb * gsize);
}

template <bool kW4A8, int kPair, int kOut, bool kQA>
__global__ void __launch_bounds__(kThreadsFor<kOut, kQA>, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb,
                   const __grid_constant__ CUtensorMap map_y, const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_l2,
                   const Params p)
{
    using C = Cfg<kPair, kOut, kQA>;
    constexpr int S = C::kStages;
    constexpr uint32_t kAcc1 = kAcc1Of<kQA>;     // accumulator slot 1's first column
    constexpr int kOvl = kOverlapOf<kQA>;        // 32-column chunks the two slots share
    constexpr int kLdb = kLdBufsOf<kQA>;         // epilogue chunk loads in flight
    constexpr int kChunks = kChunksOf<kQA>;      // 32-column chunks the epilogue drains
    constexpr int kEpiWarps = C::kEpiWarps;
    constexpr int AK = kW4A8 ? 1 : 2;  // scale atoms (128 K-elements each) per stage

    extern __shared__ __align__(1024) uint8_t smem[];
    // the swizzled tiles need a 1024-byte aligned base; both CTAs of a pair see the same
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) record_status(MXQ_ERR_UNSUPPORTED);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;                  // a stage landed (the leader's barrier counts the pair)
    uint64_t* empty = bars + S;             // a stage's MMAs completed (smem reusable)
    uint64_t* tmem_full = bars + 2 * S;     // accumulator slot complete
    uint64_t* tmem_empty = bars + 2 * S + 2;
    uint64_t* overlap_free = bars + 2 * S + 4;
    uint64_t* mma_done = bars + 2 * S + 5;
    uint64_t* sf_ready = bars + 2 * S + 6;             // [kSfBufs] scale buffer copied into TMEM
    uint64_t* sf_free = bars + 2 * S + 6 + kSfBufs;    // [kSfBufs] scale buffer's MMAs completed
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(bars + C::kNumBars);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = kPair == 2 ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int pair_id = blockIdx.x / kPair;
    const int n_pairs = gridDim.x / kPair;

    if (kPair == 2) cluster_sync();
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&map_a);
        prefetch_tmap(&map_b);
        prefetch_tmap(&map_sfa);
        prefetch_tmap(&map_sfb);
        if (kOut == kOutBf16 || (kOutEbuf<kOut> && p.write_h)) prefetch_tmap(&map_y);
        if (kOut != kOutBf16) prefetch_tmap(&map_q);
        if (p.lr_stages > 0) {
            prefetch_tmap(&map_u);
            prefetch_tmap(&map_l2);
        }
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + (kQA ? kQaWarps : 0));  // the MMAs' commit, and the A quantizer's warps
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&tmem_full[s], 1);
            mbar_init(&tmem_empty[s], kEpiWarps * kPair);
        }
        mbar_init(overlap_free, kEpiWarps * kPair);
        for (uint32_t b = 0; b < kSfBufs; ++b) {
            mbar_init(&sf_ready[b], 1);
            mbar_init(&sf_free[b], 1);
        }
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc<kPair>(tmem_base_smem, kTmemCols);
        tmem_relinquish<kPair>();
    }
    tc_fence_before();
    if (kPair == 2) cluster_sync(); else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_smem;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (each CTA)
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_last();    // weights: reused by every m-block
            const uint64_t pol_a = policy_evict_normal();  // activations: reused within a group
            constexpr uint32_t kTx = kPair * (C::kStageA + (kW4A8 ? C::kStageB / 2 : C::kStageB) +
                                              AK * 512u * 3u);
            constexpr uint32_t kTxLr = kPair * (C::kStageA + C::kRowsB * 128u);  // 128-byte rows of u and B^T
            uint32_t it = 0;
            int64_t skipped = -1;
            bool ok = true;
            for (int t = pair_id; t < p.num_tiles && ok; t += n_pairs) {
                int mb, nb;
                tile_coords<C::kGroupM>(t, p.m_blocks, p.n_blocks, mb, nb);
                for (int ks = 0; ks < p.lr_stages + p.k_stages; ++ks, ++it) {
                    const uint32_t s = it % S;
                    if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1, kWaitNs)) {
                        record_status(MXQ_ERR_TIMEOUT);
                        ok = false;
                        break;
                    }
                    if ((p.debug & 1u) && it == 0 && pair_id == 0 && leader) {
                        skipped = 0;  // deliberately leave stage 0 unfilled: the MMA wait runs out
                        continue;
                    }
                    const uint32_t bar = kPair == 2 ? mapa_shared(smem_u32(&full[s]), 0) : smem_u32(&full[s]);
                    if (kQA) fence_async_smem();  // the quantizer's reads of this stage before the copy's writes
                    if (ks < p.lr_stages) {
                        // low-rank stage: 64 columns of u as A, the same columns of B^T as B
                        if (leader) mbar_arrive_expect_tx(&full[s], kTxLr);
                        tma_load_2d<kPair>(smem + C::kOffA + s * C::kStageA, &map_u, ks * 64,
                                           mb * C::BM + static_cast<int>(rank) * 128, bar, pol_a);
                        tma_load_2d<kPair>(smem + C::kOffB + s * C::kStageB, &map_l2, ks * 64,
                                           nb * BN + static_cast<int>(rank) * C::kRowsB, bar, pol_w);
                        continue;
                    }
                    const int kq = ks - p.lr_stages;
                    if (leader) mbar_arrive_expect_tx(&full[s], kTx);
                    tma_load_2d<kPair>(smem + C::kOffA + s * C::kStageA, &map_a, kq * 128,
                                       mb * C::BM + static_cast<int>(rank) * 128, bar, pol_a);
                    tma_load_2d<kPair>(smem + C::kOffB + s * C::kStageB, &map_b, kq * 128,
                                       nb * BN + static_cast<int>(rank) * C::kRowsB, bar, pol_w);
                    tma_load_2d<kPair>(smem + C::kOffSFA + s * C::kStageSFA, &map_sfa, kq * AK * 128,
                                       mb * kPair + static_cast<int>(rank), bar, pol_a);
                    tma_load_2d<kPair>(smem + C::kOffSFB + s * C::kStageSFB, &map_sfb, kq * AK * 128,
                                       (nb * BN) / 128, bar, pol_w);
                }
            }
            // drain: the last stages' loads have landed once their consumer released them
            const uint32_t first = it > S ? it - S : 0;
            for (uint32_t i = first; i < it && ok; ++i) {
                if (static_cast<int64_t>(i) == skipped) continue;
                if (!mbar_wait(&empty[i % S], (i / S) & 1, kWaitNs)) {
                    record_status(MXQ_ERR_TIMEOUT);
                    break;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader CTA)
        if (leader && lane == 0) {
            // One thread issues everything; its instruction stream must stay well inside the
            // 128 tensor-pipe cycles an MMA takes, so all addresses are precomputed words.
            constexpr uint32_t fa = kW4A8 ? 0u : 1u;  // A element type: E4M3 (mxf8f6f4) / E2M1 (mxf4)
            constexpr uint32_t fb = kW4A8 ? 5u : 1u;  // B element type: E2M1 in both kinds
            constexpr int KPS = kW4A8 ? 128 : 256;    // K elements per stage
            constexpr int KPM = kW4A8 ? 32 : 64;      // K elements per MMA
            const uint32_t a_lo0 = sdesc_sw128_lo(smem_u32(smem + C::kOffA));
            const uint32_t b_lo0 = sdesc_sw128_lo(smem_u32(smem + C::kOffB));
            uint32_t s = 0, ph = 0;  // ring slot and phase parity of the next stage to consume
            uint32_t sfi = 0;        // stages consumed so far (selects the scale buffer)
            int tcount = 0;
            bool ok = true;
            for (int t = pair_id; t < p.num_tiles && ok; t += n_pairs, ++tcount) {
                const int slot = tcount & 1;
                const uint32_t acc = tmem_base + (slot ? kAcc1 : 0u);
                if (!mbar_wait(&tmem_empty[slot], ((tcount >> 1) & 1) ^ 1, kWaitNs) ||
                    (kOvl > 0 && tcount > 0 && !mbar_wait(overlap_free, (tcount - 1) & 1, kWaitNs))) {
                    record_status(MXQ_ERR_TIMEOUT);
                    break;
                }
                tc_fence_after();
                int mb_t, nb_t;
                tile_coords<C::kGroupM>(t, p.m_blocks, p.n_blocks, mb_t, nb_t);
                // the tile's first weight row inside its 128-aligned scale window, in 32-row columns
                const uint32_t sfb_shift = static_cast<uint32_t>(((nb_t * BN) % 128) / 32);
                for (int ks = 0; ks < p.lr_stages + p.k_stages; ++ks) {
                    if (ks < p.lr_stages) {
                        // low-rank stage: four bf16 MMAs (K = 16 each, 32 bytes of every row);
                        // the first one of the tile initializes the accumulator
                        if (!mbar_wait(&full[s], ph, kWaitNs)) {
                            record_status(MXQ_ERR_TIMEOUT);
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_lo = a_lo0 + s * (C::kStageA >> 4);
                        const uint32_t b_lo = b_lo0 + s * (C::kStageB >> 4);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_bf16<kPair>(acc, a_lo + 2 * j, b_lo + 2 * j, kSdescSw128Hi,
                                            idesc_bf16(C::BM, static_cast<uint32_t>(p.mma_n)), (ks > 0 || j > 0) ? 1u : 0u);
                        tc_commit<kPair>(&empty[s]);
                        if (++s == S) { s = 0; ph ^= 1; }
                        continue;
                    }
                    const int kq = ks - p.lr_stages;
                    const uint32_t bsf = sfi % kSfBufs;
                    if (!mbar_wait(&full[s], ph, kWaitNs) ||
                        !mbar_wait(&sf_ready[bsf], (sfi / kSfBufs) & 1, kWaitNs)) {
                        record_status(MXQ_ERR_TIMEOUT);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sft = tmem_base + kSfCol + bsf * kSfBufCols;
                    const uint32_t a_lo = a_lo0 + s * (C::kStageA >> 4);
                    const uint32_t b_lo = b_lo0 + s * (C::kStageB >> 4);
                    const int kvalid = p.K - kq * KPS;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t sf_id = kW4A8 ? static_cast<uint32_t>(j) : static_cast<uint32_t>((j & 1) * 2);
                        const uint32_t atom = kW4A8 ? 0u : static_cast<uint32_t>(j >> 1);
                        if (j * KPM < kvalid)
                            mma_block_scaled<kPair, kW4A8>(acc, a_lo + 2 * j, b_lo + 2 * j, kSdescSw128Hi,
                                                           idesc_block_scaled(fa, fb, C::BM, BN, sf_id, sf_id),
                                                           sft + 4 * atom, sft + 8 + 8 * atom + sfb_shift,
                                                           (ks > 0 || j > 0) ? 1u : 0u);  // ks counts low-rank stages
                    }
                    tc_commit<kPair>(&empty[s]);             // stage s free (in both CTAs) after these MMAs
                    tc_commit_local<kPair>(&sf_free[bsf]);  // and so is its scale buffer
                    ++sfi;
                    if (++s == S) { s = 0; ph ^= 1; }
                }
                if (!ok) break;
                tc_commit<kPair>(&tmem_full[slot]);  // accumulators ready for both CTAs' epilogues
            }
            // every MMA issued by this thread completes before TMEM is released
            tc_commit_local<kPair>(mma_done);
            if (!mbar_wait(mma_done, 0, kWaitNs)) record_status(MXQ_ERR_TIMEOUT);
        }
    } else if (warp == 2 + kEpiWarps) {
        // ------------------------------------------------------------ scale copies (leader CTA)
        // tcgen05 operations issued by one thread execute in order, so scale copies issued
        // by the MMA thread would wait for its MMAs to drain.  This thread issues them
        // instead, into kSfBufs buffers a stage or two ahead of the MMAs.
        if (leader && lane == 0) {
            const uint32_t sfa_s0 = smem_u32(smem + C::kOffSFA);
            const uint32_t sfb_s0 = smem_u32(smem + C::kOffSFB);
            uint32_t s = 0, ph = 0, sfi = 0;
            bool ok = true;
            for (int t = pair_id; t < p.num_tiles && ok; t += n_pairs) {
                for (int ks = 0; ks < p.lr_stages + p.k_stages; ++ks) {
                    if (ks < p.lr_stages) {  // low-rank stages carry no scales: keep the ring position
                        if (++s == S) { s = 0; ph ^= 1; }
                        continue;
                    }
                    const uint32_t bsf = sfi % kSfBufs;
                    if (!mbar_wait(&full[s], ph, kWaitNs) ||
                        !mbar_wait(&sf_free[bsf], ((sfi / kSfBufs) & 1) ^ 1, kWaitNs)) {
                        record_status(MXQ_ERR_TIMEOUT);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sft = tmem_base + kSfCol + bsf * kSfBufCols;
                    const uint32_t sfa_s = sfa_s0 + s * C::kStageSFA;
                    const uint32_t sfb_s = sfb_s0 + s * C::kStageSFB;
#pragma unroll
                    for (int a = 0; a < AK; ++a) {
                        tc_copy_sf_atom<kPair>(sft + 4 * a, sdesc_sf_atom(sfa_s + a * 512));
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            tc_copy_sf_atom<kPair>(sft + 8 + 8 * a + 4 * h, sdesc_sf_atom(sfb_s + (h * AK + a) * 512));
                    }
                    tc_commit_local<kPair>(&sf_ready[bsf]);  // arrives when the copies (both CTAs) completed
                    ++sfi;
                    if (++s == S) { s = 0; ph ^= 1; }
                }
            }
        }
    } else if (kQA && warp > 2 + kEpiWarps) {
        // ------------------------------------------------------------ A quantizer (kQA, lone CTA)
        // The bf16 stages' A tiles are rows of the activation, 64 channels (two MX blocks)
        // a stage.  Eight warps, two to a scheduler: thread (row, block) takes block b of
        // one of the tile's 128 rows, b by warp group.  Once a stage lands it reads its
        // block (64 bytes; 16-byte chunk q of row r sits at chunk q ^ (r & 7) under the
        // 128-byte swizzle), releases the stage (the stage's second consumer, beside the
        // MMAs), and forms the block's E8M0 scale and codes with the activation quantizer's
        // arithmetic: scale code max(0, E(amax) - emax) from the bf16 exponent field of the
        // block's abs-max (255 for a NaN or Inf), codes cvt(x 2^-s) rounded to nearest even
        // with saturation, all-zero codes under scale 255.  Rows past M (zeros from the
        // copy) write only their scale byte, 0, as the tiled layout's padding; k-blocks past
        // K / 32 get scale 0 and no codes.  One tile column (N <= 128), so every A stage is
        // seen once.
        static_assert(!kQA || (kPair == 1 && kOut == kOutBf16 && !kW4A8), "A quantizer: bf16 lone-CTA kernel only");
        const int qw = warp - 3 - kEpiWarps;
        const int r_in = (qw & 3) * 32 + lane;  // row within the tile
        const uint32_t b = static_cast<uint32_t>(qw >> 2);  // which of a stage's two blocks
        const uint32_t sw = static_cast<uint32_t>(r_in & 7);
        const bool e4m3 = p.qa_fmt == kFmtE4M3;
        const uint32_t emax = e4m3 ? 8u : 2u;
        const uint32_t KB = static_cast<uint32_t>(p.K / 32);
        const uint32_t kb_pad = 4u * p.qa_atoms_k;
        const size_t row_bytes = e4m3 ? static_cast<size_t>(p.K) : static_cast<size_t>(p.K / 2);
        uint32_t s = 0, ph = 0;
        bool ok = true;
        for (int t = pair_id; t < p.num_tiles && ok; t += n_pairs) {
            int mb, nb;
            tile_coords<C::kGroupM>(t, p.m_blocks, p.n_blocks, mb, nb);
            const uint32_t row = static_cast<uint32_t>(mb * C::BM + r_in);
            const bool live = static_cast<int>(row) < p.M;
            // this row's scale bytes: atom row block, 32-row column inside the atom
            uint8_t* sf_row = p.qa_sf + static_cast<size_t>(row >> 7) * p.qa_atoms_k * 512u + (row & 31u) * 16u +
                              ((row >> 5) & 3u) * 4u;
            uint8_t* code_row = p.qa_codes + static_cast<size_t>(row) * row_bytes;
            for (int ks = 0; ks < p.lr_stages; ++ks) {
                const bool landed = mbar_wait(&full[s], ph, kWaitNs);
                if (!__all_sync(0xFFFFFFFFu, landed)) {
                    if (lane == 0) record_status(MXQ_ERR_TIMEOUT);
                    ok = false;
                    break;
                }
                const uint8_t* rowp = smem + C::kOffA + s * C::kStageA + r_in * 128;
                uint32_t w[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v =
                        *reinterpret_cast<const uint4*>(rowp + 16u * ((4u * b + static_cast<uint32_t>(q)) ^ sw));
                    w[4 * q] = v.x;
                    w[4 * q + 1] = v.y;
                    w[4 * q + 2] = v.z;
                    w[4 * q + 3] = v.w;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (++s == S) { s = 0; ph ^= 1; }
                const uint32_t kb = 2u * static_cast<uint32_t>(ks) + b;
                if (ks == p.lr_stages - 1 && b == 0)  // the layout's padding k-blocks past the last stage
                    for (uint32_t kp = kb + 2u; kp < kb_pad; kp += 2u)
                        *reinterpret_cast<uint16_t*>(sf_row + (kp >> 2) * 512u + (kp & 3u)) = 0;
                if (kb >= KB) {  // past K: scale 0, no codes
                    sf_row[(kb >> 2) * 512u + (kb & 3u)] = 0;
                    continue;
                }
                uint32_t m2 = absmax_bf16x2(absmax_bf16x2(w[0], w[1]), absmax_bf16x2(w[2], w[3]));
#pragma unroll
                for (int i = 4; i < 16; i += 4)
                    m2 = absmax_bf16x2(m2, absmax_bf16x2(absmax_bf16x2(w[i], w[i + 1]), absmax_bf16x2(w[i + 2], w[i + 3])));
                m2 = absmax_bf16x2(m2, __byte_perm(m2, 0, 0x1032));
                const uint32_t eb = (m2 & 0x7FFFu) >> 7;  // bf16 and E8M0 share the bias 127
                const uint32_t sc = eb == 255u ? 255u : (eb > emax ? eb - emax : 0u);
                sf_row[(kb >> 2) * 512u + (kb & 3u)] = static_cast<uint8_t>(sc);
                if (!live) continue;
                const float inv = __uint_as_float((254u - min(sc, 253u)) << 23);  // 2^(127 - sc)
                const float2 inv2 = make_float2(inv, inv);
                const uint32_t keep = sc == 255u ? 0u : 0xFFFFFFFFu;
                if (e4m3) {
                    uint32_t c4[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float2 f0 = __fmul2_rn(make_float2(lo_f(w[2 * i]), hi_f(w[2 * i])), inv2);
                        const float2 f1 = __fmul2_rn(make_float2(lo_f(w[2 * i + 1]), hi_f(w[2 * i + 1])), inv2);
                        c4[i] = (cvt_e4m3x2(f0.x, f0.y) | (cvt_e4m3x2(f1.x, f1.y) << 16)) & keep;
                    }
                    uint4* d4 = reinterpret_cast<uint4*>(code_row + kb * 32u);
                    __stcs(d4, make_uint4(c4[0], c4[1], c4[2], c4[3]));
                    __stcs(d4 + 1, make_uint4(c4[4], c4[5], c4[6], c4[7]));
                } else {
                    uint32_t c2[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float q[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __fmul2_rn(make_float2(lo_f(w[4 * i + e]), hi_f(w[4 * i + e])), inv2);
                            q[2 * e] = f.x;
                            q[2 * e + 1] = f.y;
                        }
                        c2[i] = cvt_e2m1x8(q) & keep;
                    }
                    __stcs(reinterpret_cast<uint4*>(code_row + kb * 16u), make_uint4(c2[0], c2[1], c2[2], c2[3]));
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (each CTA)
        // Each warp owns the 32 TMEM lanes (= output rows) of its quarter.  Per tile it
        // drains the accumulator in 32-column chunks: the load of chunk c+1 is in flight
        // while chunk c gets its bias, is rounded to bf16, staged (64-byte swizzle) and
        // written by a TMA store.  The shared columns go first; the slot is handed back to
        // the MMA issuer as soon as its last chunk is in registers.
        const uint64_t pol_y = policy_evict_first();
        const int ew = warp - 2;
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const uint32_t lanes = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        uint8_t* ebuf0 = smem + C::kOffEpi + ew * 2 * kEpiBuf;
        uint8_t* qbuf0 = smem + C::kOffQ + ew * C::kQBufs * C::kQBuf;
        const uint16_t* lut = reinterpret_cast<const uint16_t*>(smem + C::kOffLut);
        if constexpr (kOut != kOutBf16) {
            // the GELU table, built by the epilogue warps while the first tile's MMAs run
            if (p.gelu)
                gelu_table_fill(reinterpret_cast<uint16_t*>(smem + C::kOffLut), threadIdx.x - 64u, kEpiWarps * 32u);
            named_bar_sync(1, kEpiWarps * 32);
        }
        const uint32_t bar_overlap = kPair == 2 ? mapa_shared(smem_u32(overlap_free), 0) : smem_u32(overlap_free);
        const bool has_bias = p.bias != nullptr;
        int eb = 0;
        int tcount = 0;
        for (int t = pair_id; t < p.num_tiles; t += n_pairs, ++tcount) {
            const int slot = tcount & 1;
            int mb, nb;
            tile_coords<C::kGroupM>(t, p.m_blocks, p.n_blocks, mb, nb);
            // this lane's 8 bias values (tile columns 8*lane ..), loaded before the wait so
            // the load latency hides behind the tile's MMAs; chunks fetch them by shuffle
            uint4 bias8 = make_uint4(0u, 0u, 0u, 0u);
            const int nbias = nb * BN + 8 * lane;
            if (has_bias && nbias + 8 <= p.N) bias8 = __ldg(reinterpret_cast<const uint4*>(p.bias + nbias));
            const bool waited = mbar_wait(&tmem_full[slot], (tcount >> 1) & 1, kWaitNs);
            if (!__all_sync(0xFFFFFFFFu, waited)) {  // the warp leaves together (tcgen05.ld is .aligned)
                if (lane == 0) record_status(MXQ_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();
            const uint32_t col0 = slot ? kAcc1 : 0u;
            const int row0 = mb * C::BM + static_cast<int>(rank) * 128 + q * 32;
            const uint32_t tmem_empty_bar = kPair == 2 ? mapa_shared(smem_u32(&tmem_empty[slot]), 0)
                                                       : smem_u32(&tmem_empty[slot]);
            // chunk order: slot 0 drains its shared (top) columns first, slot 1 its bottom ones
            auto chunk_of = [&](int ci) {
                return slot ? ci : (ci < kOvl ? BN / 32 - kOvl + ci : ci - kOvl);
            };
            // after the loads of this warp's chunks up to drain index ci have landed:
            // release what the MMA issuer waits for (every epilogue warp arrives on both)
            auto landed = [&](int ci, int last_shared, int last) {
                if (ci == last_shared || ci == last) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(ci == last ? tmem_empty_bar : bar_overlap);
                }
            };
            // a ring of kLdBufs chunk registers: the first kLdBufs loads go out back to back, so
            // the shared columns (kOverlapChunks <= kLdBufs chunks) are released after one wait
            // one 32-column chunk (the ci-th in drain order) whose accumulators are in acc
            auto process = [&](const uint32_t(&acc)[32], int ci) __attribute__((always_inline)) {
                const int c = chunk_of(ci);
                uint32_t sc_byte = 0u;  // quantizing epilogue: the chunk's E8M0 scale
                const int n = nb * BN + c * 32;
                if (n < p.N) {  // warp-uniform
                    // the chunk's 32 bias values as 16 bf16 pairs (columns 2i, 2i + 1 in word
                    // i), kept packed and widened where they are used
                    uint32_t bw[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) bw[i] = 0u;
                    if (has_bias) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const int src = 4 * c + g;  // lane holding columns c*32 + 8g ..
                            bw[4 * g] = __shfl_sync(0xFFFFFFFFu, bias8.x, src);
                            bw[4 * g + 1] = __shfl_sync(0xFFFFFFFFu, bias8.y, src);
                            bw[4 * g + 2] = __shfl_sync(0xFFFFFFFFu, bias8.z, src);
                            bw[4 * g + 3] = __shfl_sync(0xFFFFFFFFu, bias8.w, src);
                        }
                    }
                    // o: the chunk in bf16 -- y = acc + bias, or h = GELU of that rounded to bf16
                    uint32_t o[16];
                    const float2 alpha2 = make_float2(p.alpha, p.alpha);
                    // the activation choice is taken once per chunk, outside the unrolled
                    // loops, so that the 16 independent GELU chains interleave
                    auto chunk_out = [&](auto gelu) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float2 y = __ffma2_rn(
                                make_float2(__uint_as_float(acc[2 * i]), __uint_as_float(acc[2 * i + 1])), alpha2,
                                make_float2(lo_f(bw[i]), hi_f(bw[i])));
                            __nv_bfloat162 y2 = __floats2bfloat162_rn(y.x, y.y);
                            const uint32_t w = *reinterpret_cast<uint32_t*>(&y2);
                            if constexpr (decltype(gelu)::value)
                                o[i] = gelu_bf16_bits(w & 0xFFFFu, lut) | (gelu_bf16_bits(w >> 16, lut) << 16);
                            else
                                o[i] = w;
                        }
                    };
                    if (kOut != kOutBf16 && p.gelu)
                        chunk_out(std::true_type{});
                    else
                        chunk_out(std::false_type{});
                    const bool store_y = kOut == kOutBf16 || (kOutEbuf<kOut> && p.write_h);
                    uint8_t* buf = ebuf0 + eb * kEpiBuf;
                    // the stores that last used this chunk's buffers have read them
                    if (lane == 0) {
                        if constexpr (C::kQBufs == 1)
                            bulk_wait_read<0>();
                        else
                            bulk_wait_read<1>();
                    }
                    __syncwarp();
                    if (store_y) {
                        const uint32_t rsw = (static_cast<uint32_t>(lane) >> 1) & 3u;
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch) {
                            uint4* dst = reinterpret_cast<uint4*>(buf + lane * 64 + ((ch ^ rsw) * 16));
                            *dst = make_uint4(o[4 * ch], o[4 * ch + 1], o[4 * ch + 2], o[4 * ch + 3]);
                        }
                    }
                    if constexpr (kOut != kOutBf16) {
                        // this lane's 32 values are one MX block of the next layer's K: its
                        // E8M0 scale and element codes, rounded to nearest even by cvt
                        constexpr uint32_t kEmax = kOutE4M3<kOut> ? 8u : 2u;
                        uint32_t m2 = o[0];
#pragma unroll
                        for (int i = 1; i < 16; ++i) m2 = absmax_bf16x2(m2, o[i]);
                        m2 = absmax_bf16x2(m2, __byte_perm(m2, 0, 0x1032));
                        const uint32_t sc = e8m0_code<kEmax>(m2);
                        const float inv = e8m0_inverse(sc);
                        const uint32_t keep = sc == 255u ? 0u : 0xFFFFFFFFu;  // a non-finite block: codes 0
                        uint8_t* qb = qbuf0 + (C::kQBufs == 2 ? eb : 0) * C::kQBuf;
                        if constexpr (!kOutE4M3<kOut>) {
                            uint32_t cw[4];
                            const float2 inv2 = make_float2(inv, inv);
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                float v[8];
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const float2 f = __fmul2_rn(make_float2(lo_f(o[4 * k + i]), hi_f(o[4 * k + i])), inv2);
                                    v[2 * i] = f.x;
                                    v[2 * i + 1] = f.y;
                                }
                                cw[k] = cvt_e2m1x8(v) & keep;
                            }
                            *reinterpret_cast<uint4*>(qb + lane * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
                        } else {
                            uint32_t cw[8];
                            const float2 inv2 = make_float2(inv, inv);
#pragma unroll
                            for (int k = 0; k < 8; ++k) {
                                const float2 f0 = __fmul2_rn(make_float2(lo_f(o[2 * k]), hi_f(o[2 * k])), inv2);
                                const float2 f1 = __fmul2_rn(make_float2(lo_f(o[2 * k + 1]), hi_f(o[2 * k + 1])), inv2);
                                cw[k] = (cvt_e4m3x2(f0.x, f0.y) | (cvt_e4m3x2(f1.x, f1.y) << 16)) & keep;
                            }
                            *reinterpret_cast<uint4*>(qb + lane * 32) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
                            *reinterpret_cast<uint4*>(qb + lane * 32 + 16) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
                        }
                        sc_byte = sc;
                    }
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if (store_y) tma_store_2d(&map_y, buf, n, row0, pol_y);
                        if constexpr (kOut != kOutBf16)
                            tma_store_2d(&map_q, qbuf0 + (C::kQBufs == 2 ? eb : 0) * C::kQBuf,
                                         kOutE4M3<kOut> ? n : n / 2, row0,
                                         pol_y);
                        bulk_commit();
                    }
                    eb ^= 1;
                }
                if constexpr (kOut != kOutBf16) {
                    // this row's scale byte of k-block nb*8 + c, straight into the tiled
                    // layout; rows between M and the 128-row padding, and k-blocks past N
                    // inside the padding, get 0 as the layout requires
                    const int row = row0 + lane;
                    const uint32_t kb = static_cast<uint32_t>(nb) * 8u + static_cast<uint32_t>(c);
                    if (row < p.q_rows_pad && kb < 4u * p.q_atoms_k) {
                        const size_t off = (static_cast<size_t>(row >> 7) * p.q_atoms_k + (kb >> 2)) * 512u +
                                           (row & 31) * 16u + ((row >> 5) & 3) * 4u + (kb & 3u);
                        p.q_sf[off] = row < p.M ? static_cast<uint8_t>(sc_byte) : uint8_t(0);
                    }
                }
            };
            if constexpr (kOut == kOutBf16) {
                // a ring of kLdBufs chunk registers, fully unrolled: the first kLdBufs loads go
                // out back to back, so the shared columns are released after one wait
                uint32_t r[kLdb][32];
#pragma unroll
                for (int j = 0; j < kLdb; ++j) tmem_ld_x32(lanes + col0 + chunk_of(j) * 32, r[j]);
                int issued = kLdb, landed_upto = 0;  // constants once the loop below is unrolled
#pragma unroll
                for (int ci = 0; ci < kChunks; ++ci) {
                    if (ci >= landed_upto) {  // everything issued so far lands together
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < kChunks; ++j)
                            if (j >= landed_upto && j < issued) {
                                tmem_regs_ready(r[j % kLdb]);
                                landed(j, kOvl - 1, kChunks - 1);
                            }
                        landed_upto = issued;
                    }
                    process(r[ci % kLdb], ci);
                    if (ci + kLdb < kChunks) {  // refill the buffer just drained
                        tmem_ld_x32(lanes + col0 + chunk_of(ci + kLdb) * 32, r[ci % kLdb]);
                        issued = ci + kLdb + 1;
                    }
                }
            } else {
                // Two warps per lane quarter take alternate chunks of the drain order (the
                // first group, warps 2-5, even ones; warps 6-9 odd ones), so the three shared
                // chunks split 2 + 1 and each warp frees them after its first two loads.  The
                // chunk body is long (GELU of 32 values), so the loop stays rolled, with a
                // two-chunk register ring advanced by moves.
                static_assert(BN / 32 == 8 && kOverlapChunks == 3 && C::kEpiWarps == 8, "chunk split");
                const int grp = ew >> 2;
                constexpr int kMine = 4;
                const int last_shared = grp == 0 ? 1 : 0;  // local index of its last shared chunk
                uint32_t ra[32], rb[32];
                tmem_ld_x32(lanes + col0 + chunk_of(grp) * 32, ra);
                tmem_ld_x32(lanes + col0 + chunk_of(grp + 2) * 32, rb);
                tmem_ld_wait();
                tmem_regs_ready(ra);
                tmem_regs_ready(rb);
                landed(0, last_shared, kMine - 1);
                landed(1, last_shared, kMine - 1);
#pragma unroll 1
                for (int i = 0; i < kMine; ++i) {
                    process(ra, grp + 2 * i);
                    if (i + 1 < kMine) {
                        if (i >= 1) {  // chunk i+1, loaded during this chunk's work
                            tmem_ld_wait();
                            tmem_regs_ready(rb);
                            landed(i + 1, last_shared, kMine - 1);
                        }
#pragma unroll
                        for (int k = 0; k < 32; ++k) ra[k] = rb[k];
                        if (i + 2 < kMine) tmem_ld_x32(lanes + col0 + chunk_of(grp + 2 * (i + 2)) * 32, rb);
                    }
                }
            }
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    if (kPair == 2) cluster_sync(); else __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc<kPair>(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------- host

uint32_t g_debug_flags = 0;

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
                 uint64_t stride_bytes, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {d0, d1};
    const cuuint64_t strides[1] = {stride_bytes};
    const cuuint32_t box[2] = {b0, b1};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

void set_debug_flags(uint32_t flags) { g_debug_flags = flags; }
uint32_t debug_flags() { return g_debug_flags; }

int read_and_clear_device_status(cudaStream_t stream, uint32_t* out)
{
    uint32_t v = 0, zero = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MXQ_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return MXQ_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero) != cudaSuccess) return MXQ_ERR_CUDA;
    *out = v;
    return MXQ_OK;
}

namespace {

template <bool kW4A8, int kPair, int kOut, bool kQA = false>
cudaError_t launch_variant(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& msa,
                           const CUtensorMap& msb, const CUtensorMap& my, const CUtensorMap& mq,
                           const CUtensorMap& mu, const CUtensorMap& ml, const Params& p, int grid,
                           cudaStream_t stream)
{
    using C = Cfg<kPair, kOut, kQA>;
    auto kern = mx_gemm_kernel<kW4A8, kPair, kOut, kQA>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kThreadsFor<kOut, kQA>, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kPair;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = kPair == 2 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, ma, mb, msa, msb, my, mq, mu, ml, p);
}

template <bool kW4A8, int kPair>
cudaError_t launch_out(int out, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& msa,
                       const CUtensorMap& msb, const CUtensorMap& my, const CUtensorMap& mq, const CUtensorMap& mu,
                       const CUtensorMap& ml, const Params& p, int grid, cudaStream_t stream)
{
    if (out == kOutGeluE2M1)
        return launch_variant<kW4A8, kPair, kOutGeluE2M1>(ma, mb, msa, msb, my, mq, mu, ml, p, grid, stream);
    if (out == kOutGeluE4M3)
        return launch_variant<kW4A8, kPair, kOutGeluE4M3>(ma, mb, msa, msb, my, mq, mu, ml, p, grid, stream);
    if (out == kOutQE2M1)
        return launch_variant<kW4A8, kPair, kOutQE2M1>(ma, mb, msa, msb, my, mq, mu, ml, p, grid, stream);
    if (out == kOutQE4M3)
        return launch_variant<kW4A8, kPair, kOutQE4M3>(ma, mb, msa, msb, my, mq, mu, ml, p, grid, stream);
    return launch_variant<kW4A8, kPair, kOutBf16>(ma, mb, msa, msb, my, mq, mu, ml, p, grid, stream);
}

}  // namespace

int launch_gemm(const GemmArgs& g, cudaStream_t stream, const char** msg, char* path, size_t path_len)
{
    const bool bf16 = g.bf16;
    const bool w4a8 = !bf16 && g.a_fmt == kFmtE4M3;
    const bool quant_out = g.out_fmt >= 0;
    const bool quant_a = bf16 && g.qa_fmt >= 0;
    if (quant_a && (g.N > 128 || quant_out || g.qa_codes == nullptr || g.qa_sf == nullptr)) {
        *msg = "quantizing A beside a bf16 GEMM needs N <= 128, a bf16 output and both MX buffers";
        return MXQ_ERR_INVALID_ARG;
    }
    // CTA pairs for anything taller than one 128-row tile; a lone CTA otherwise, and for the
    // bf16 GEMM that quantizes its A (each CTA's quantizer waits on its own stage barriers,
    // where a pair's loads all complete on the leader's).
    const int pair = g.M > 128 && !quant_a ? 2 : 1;
    const int rows_b = BN / pair;
    const int64_t atoms_k = sf_atoms_k(g.K);
    const int ak = w4a8 ? 1 : 2;
    CUtensorMap ma, mb, msa, msb, my, mq, mu, ml;
    bool ok = true;
    if (!bf16) {
        const uint64_t a_row = w4a8 ? g.K : g.K / 2;
        ok = make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a_codes, a_row, g.M, a_row, 128, 128,
                         CU_TENSOR_MAP_SWIZZLE_128B);
        if (w4a8)
            ok = ok && make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, g.w_codes, g.K, g.N, g.K / 2, 128,
                                   rows_b, CU_TENSOR_MAP_SWIZZLE_128B);
        else
            ok = ok && make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.w_codes, g.K / 2, g.N, g.K / 2, 128, rows_b,
                                   CU_TENSOR_MAP_SWIZZLE_128B);
        // scale atoms as 32-bit words: one 2-D row of atoms_k*128 words per 128-row tile
        ok = ok && make_map_2d(&msa, CU_TENSOR_MAP_DATA_TYPE_UINT32, g.a_sf, atoms_k * 128, ceil_div(g.M, 128),
                               atoms_k * 512, ak * 128, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
        ok = ok && make_map_2d(&msb, CU_TENSOR_MAP_DATA_TYPE_UINT32, g.w_sf, atoms_k * 128, ceil_div(g.N, 128),
                               atoms_k * 512, ak * 128, 2, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    // bf16 output (y, or h of the quantizing epilogue): 32 x 32 boxes, 64-byte swizzle
    const void* ybase = g.y ? g.y : g.q_codes;  // without h the map is never used
    ok = ok && make_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ybase, g.N, g.M, g.N * 2, 32, 32,
                           CU_TENSOR_MAP_SWIZZLE_64B);
    if (quant_out) {
        // codes of the quantized output: one 32-element block (16 or 32 bytes) x 32 rows per box
        const uint64_t q_row = g.out_fmt == kFmtE4M3 ? g.N : g.N / 2;
        ok = ok && make_map_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.q_codes, q_row, g.M, q_row,
                               g.out_fmt == kFmtE4M3 ? 32 : 16, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
    } else {
        mq = my;  // never used by the bf16 epilogue
    }
    // bf16 stages (the low-rank branch, or every stage of a plain bf16 GEMM): operands bf16
    // and K-major, one 64-element (128-byte) column block per stage as the A and B tiles of
    // a stage; a K that is not a multiple of 64 reads zeros past its end
    const int64_t lr_k = bf16 ? g.K : g.lr_rank;
    const void* lr_a = bf16 ? g.a_codes : g.lr_u;
    const void* lr_b = bf16 ? g.w_codes : g.lr_l2t;
    const int lr_stages = lr_k > 0 ? static_cast<int>(ceil_div(lr_k, 64)) : 0;
    if (lr_stages > 0) {
        ok = ok && make_map_2d(&mu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lr_a, lr_k, g.M, lr_k * 2, 64, 128,
                               CU_TENSOR_MAP_SWIZZLE_128B);
        ok = ok && make_map_2d(&ml, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lr_b, lr_k, g.N, lr_k * 2, 64,
                               quant_a ? 128 : rows_b, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (bf16) {
        ma = msa = mu;  // never used without block-scaled stages
        mb = msb = ml;
    } else if (lr_stages == 0) {
        mu = ma;  // never used without bf16 stages
        ml = mb;
    }
    if (!ok) {
        *msg = "cuTensorMapEncodeTiled failed (driver entry point unavailable or invalid operand layout)";
        return MXQ_ERR_CUDA;
    }
    Params p;
    p.bias = static_cast<const __nv_bfloat16*>(g.bias);
    p.M = static_cast<int>(g.M);
    p.N = static_cast<int>(g.N);
    p.K = static_cast<int>(g.K);
    p.m_blocks = static_cast<int>(ceil_div(g.M, 128 * pair));
    p.n_blocks = static_cast<int>(ceil_div(g.N, BN));
    p.num_tiles = p.m_blocks * p.n_blocks;
    p.k_stages = bf16 ? 0 : static_cast<int>(ceil_div(g.K, w4a8 ? 128 : 256));
    p.debug = g_debug_flags;
    p.q_sf = static_cast<uint8_t*>(g.q_sf);
    p.q_atoms_k = quant_out ? static_cast<uint32_t>(sf_atoms_k(g.N)) : 0u;
    p.q_rows_pad = static_cast<int>(ceil_div(g.M, 128) * 128);
    p.write_h = quant_out && g.y != nullptr ? 1 : 0;
    p.gelu = g.out_gelu ? 1 : 0;
    p.alpha = g.alpha;
    p.lr_stages = lr_stages;
    // a lone CTA's only tile column: bf16 MMAs as wide as the output (rounded up to 16, the
    // M = 128 granule), not the tile's 256 columns; a pair's MMA of another width would
    // take a different set of B rows from each CTA, so pairs keep 256
    p.mma_n = bf16 && pair == 1 && p.n_blocks == 1 ? static_cast<int>((g.N + 15) / 16 * 16) : BN;
    p.qa_codes = static_cast<uint8_t*>(g.qa_codes);
    p.qa_sf = static_cast<uint8_t*>(g.qa_sf);
    p.qa_atoms_k = quant_a ? static_cast<uint32_t>(sf_atoms_k(g.K)) : 0u;
    p.qa_fmt = quant_a ? g.qa_fmt : -1;
    const int out = !quant_out  ? kOutBf16
                    : p.write_h ? (g.out_fmt == kFmtE4M3 ? kOutGeluE4M3 : kOutGeluE2M1)
                                : (g.out_fmt == kFmtE4M3 ? kOutQE4M3 : kOutQE2M1);

    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(p.num_tiles, sms / pair) * pair;
    cudaError_t e;
    if (quant_a)
        e = launch_variant<false, 1, kOutBf16, true>(ma, mb, msa, msb, my, mq, mu, ml, p, grid, stream);
    else if (w4a8)
        e = pair == 2 ? launch_out<true, 2>(out, ma, mb, msa, msb, my, mq, mu, ml, p, grid, stream)
                      : launch_out<true, 1>(out, ma, mb, msa, msb, my, mq, mu, ml, p, grid, stream);
    else
        e = pair == 2 ? launch_out<false, 2>(out, ma, mb, msa, msb, my, mq, mu, ml, p, grid, stream)
                      : launch_out<false, 1>(out, ma, mb, msa, msb, my, mq, mu, ml, p, grid, stream);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) {
        *msg = cudaGetErrorString(e);
        return MXQ_ERR_CUDA;
    }
    if (path && bf16)
        snprintf(path, path_len, "bf16 kind::f16 %s %dx%d (mma n %d) grid %d tiles %d%s", pair == 2 ? "2cta" : "1cta",
                 128 * pair, BN, p.mma_n, grid, p.num_tiles,
                 quant_a ? (g.qa_fmt == kFmtE4M3 ? " +quantize a->e4m3" : " +quantize a->e2m1") : "");
    else if (path)
        snprintf(path, path_len, "native %s %s %dx%d grid %d tiles %d%s%s", w4a8 ? "mxf8f6f4" : "mxf4",
                 pair == 2 ? "2cta" : "1cta", 128 * pair, BN, grid, p.num_tiles,
                 !quant_out ? "" : g.out_gelu ? (g.out_fmt == kFmtE4M3 ? " +gelu->e4m3" : " +gelu->e2m1")
                                              : (g.out_fmt == kFmtE4M3 ? " +quant->e4m3" : " +quant->e2m1"),
                 lr_stages ? " +lowrank(bf16 f16-mma)" : "");
    return MXQ_OK;
}

}  // namespace mxq
