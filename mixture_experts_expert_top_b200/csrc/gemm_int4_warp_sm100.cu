// gemm_int4_warp_sm100.cu -- the W4A16 down GEMM for few tokens per expert:
// int4 weights decoded straight into the A fragments of warp-level MMAs.
//
// Same result as grouped_gemm_int4_kernel's down GEMM (InfiniLM PR #500
// Qwen3-MoE report, §2.2 step 2; weights w = bf16_rne(q * scale) with one
// bf16 scale per 128 K, FlashInfer PR #7196 analysis §2, W4A16 grouped GEMM;
// fp32 accumulation):
//   y[r, h] = bf16( act[r] . W_d[e, h] )
//
// Why a second W4A16 kernel. With about 8 tokens per expert (decode), a
// tcgen05 MMA has N = 16 and costs its fixed ~45 cycles per 128 x 16 weight
// block however few tokens there are, and the decoded weights must first be
// stored into TMEM for the MMA to read them; those stores slow the MMAs
// further. Here each decoded bf16x2 register IS the MMA's operand: a warp
// decodes the packed words it needs and issues mma.sync.m16n8k16 with N = 8
// tokens, so decoded weights never leave the registers and the tensor-core
// work per weight follows the tokens present. Measured on a B200 at the W4A16
// decode shape this runs the down GEMM 15% faster than the TMEM kernel; the
// same design for gate/up (8 gate and the matching 8 up rows per MMA) was 4%
// slower than the TMEM kernel there, so gate/up stays on tcgen05.
//
// Layout of the work:
//  - Tile = (expert, 128 output features, block of up to 32 token rows), the
//    tile list of the other weights-on-M kernels. Two CTAs per SM, each a
//    producer warp and 8 MMA warps; MMA warp w owns output rows 16w .. 16w+15
//    of the tile (one m16 MMA tile).
//  - A ring stage covers K = 256: the packed weight rows (128 bytes each,
//    128-byte swizzle) by TMA, and the token rows of four 64-K quarters,
//    copied by the producer warp's 32 lanes with cp.async (one 512-byte row
//    per instruction), completing on the same mbarrier. A TMA gather of 4
//    rows per instruction would keep the TMA unit busier than the weight
//    stream itself at these row counts.
//  - Fragment mapping. m16n8k16 thread (g, c) (g = lane / 4, c = lane % 4)
//    holds MMA rows g and g + 8; here those are weight rows 2g and 2g + 1 of
//    the warp's 16, so a thread's two output features are adjacent and store
//    as one word, and the warp's 64-bit weight loads hit distinct banks under
//    the 128-byte swizzle. The MMA's K order is free as long as A and B
//    agree: in 64-K quarter Q the thread takes K = 64Q + 16c + [0, 16), which
//    is 8 packed bytes per row (one 64-bit shared load) and two 16-byte token
//    chunks; word j of those 8 bytes decodes (dequant_word) into the four K
//    pairs of chunk j, which feed two consecutive MMAs.
//  - Every wait is bounded; a timeout raises the device flag and unwinds.
#include "gemm_common.cuh"
#include "launch_util.cuh"


namespace moe {
namespace {

using namespace gemm;

constexpr int kWarpMmaWarps = 8;                    // MMA warps per CTA (one 16-row MMA tile each)
constexpr int kWarpMmaThreads = 32 * (1 + kWarpMmaWarps);
constexpr int kWarpBN = 32;                         // token rows per tile at most

template <int STAGES>
struct Int4WarpCfg {
    static constexpr int kFeat = 16 * kWarpMmaWarps;                    // 128 output features per CTA tile
    static constexpr int kABytes = kFeat * 128;                         // packed weights of a stage (K = 256)
    static constexpr int kBQuarter = kWarpBN * kBK * 2;                 // token rows of one 64-K quarter
    static constexpr int kStageBytes = kABytes + kQuarters * kBQuarter;
    static constexpr int kRingBytes = STAGES * kStageBytes;
    static constexpr int kNumBars = 2 * STAGES;
    static constexpr int kSmemBytes = 1024 + kRingBytes + 8 * kNumBars + 64 + 2 * (kMaxExperts + 1) * 4;
    static constexpr int kNB = kWarpBN / 8;                             // 8-token MMA blocks per tile at most
    static_assert(kStageBytes % 1024 == 0 && kBQuarter % 1024 == 0 && kABytes % 1024 == 0,
                  "tiles must keep 1024-byte alignment (128-byte swizzle atoms)");
    // two CTAs share an SM's 228 KB (1 KB of each CTA's is reserved)
    static_assert(2 * (kSmemBytes + 1024) <= 233472, "shared memory for two CTAs per SM");
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes 16 zero
// bytes and reads nothing.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Arrival on the mbarrier once every cp.async this thread has issued so far
// has landed; counts as one of the barrier's expected arrivals.
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint2 lds64(const uint8_t *p) { return *reinterpret_cast<const uint2 *>(p); }
__device__ __forceinline__ uint4 lds128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }

// Per-thread byte offsets of an MMA warp's shared-memory operands in a ring
// stage (fixed for the kernel's life).
struct W4LaneOffsets {
    // 8 packed bytes of quarter Q of MMA row g (rr = 0) and g + 8 (rr = 1):
    // a0[rr] + ((32 Q) ^ ax[rr]), the 128-byte swizzle folded into ax
    int a0[2], ax[2];
    int b[2];               // token row g's 16-byte chunk 2c + pp of quarter 0 (+ Q quarters, + 8 rows per block)
};

// The K loop of one tile for an MMA warp with NB 8-token blocks: KS ring
// stages, each decoded and multiplied into acc[0..NB). Scales of stage ks+1
// are fetched while stage ks runs. Returns false if a wait gave up.
template <int STAGES, int NB>
__device__ __forceinline__ bool mma_tile(const uint8_t *ring, uint64_t *full_bar, uint64_t *empty_bar, int &stage,
                                         uint32_t &sphase, int KS, const W4LaneOffsets &L, const uint16_t *srow0,
                                         const uint16_t *srow1, bool s_ok, int kgroups, volatile int *abort_flag,
                                         int *err, float (&acc)[kWarpBN / 8][4]) {
    using C = Int4WarpCfg<STAGES>;
    const int lane = threadIdx.x & 31;
    // The two 128-K groups of stage ks of both rows, group 2ks in the low
    // half and 2ks+1 in the high half. With an even number of groups per row
    // the pair is one aligned 32-bit word (scales are 4-byte aligned), loaded
    // a stage before its first use so that the load's latency hides behind a
    // stage of decoding.
    const bool pair_words = (kgroups & 1) == 0;
    auto load_scales = [&](int ks, uint32_t &d0, uint32_t &d1) {
        const int grp = 2 * ks;
        const bool ok0 = s_ok && grp < kgroups, ok1 = s_ok && grp + 1 < kgroups;
        if (pair_words) {
            d0 = ok0 ? __ldg(reinterpret_cast<const uint32_t *>(srow0 + grp)) : 0u;
            d1 = ok0 ? __ldg(reinterpret_cast<const uint32_t *>(srow1 + grp)) : 0u;
        } else {
            d0 = (ok0 ? __ldg(srow0 + grp) : 0u) | (ok1 ? static_cast<uint32_t>(__ldg(srow0 + grp + 1)) << 16 : 0u);
            d1 = (ok0 ? __ldg(srow1 + grp) : 0u) | (ok1 ? static_cast<uint32_t>(__ldg(srow1 + grp + 1)) << 16 : 0u);
        }
    };
    uint32_t nx0, nx1;
    load_scales(0, nx0, nx1);
    for (int ks = 0; ks < KS; ++ks) {
        const uint32_t sc0 = nx0, sc1 = nx1;
        if (ks + 1 < KS) load_scales(ks + 1, nx0, nx1);
        if (!mbar_wait(&full_bar[stage], sphase, abort_flag, err, 0)) return false;
        const uint8_t *st = ring + stage * C::kStageBytes;
        const uint8_t *sb = st + C::kABytes;
#pragma unroll
        for (int Q = 0; Q < kQuarters; ++Q) {
            // 8 packed bytes (K = 64Q + 16c + [0, 16)) of each of the two rows
            const uint2 w0 = lds64(st + L.a0[0] + ((32 * Q) ^ L.ax[0]));
            const uint2 w1 = lds64(st + L.a0[1] + ((32 * Q) ^ L.ax[1]));
            // the scale of group 2ks + Q/2 in both halves
            const uint32_t sel = Q < 2 ? 0x1010u : 0x3232u;
            const uint32_t sv0 = __byte_perm(sc0, 0u, sel), sv1 = __byte_perm(sc1, 0u, sel);
            const __nv_bfloat162 s20 = *reinterpret_cast<const __nv_bfloat162 *>(&sv0);
            const __nv_bfloat162 s21 = *reinterpret_cast<const __nv_bfloat162 *>(&sv1);
#pragma unroll
            for (int pp = 0; pp < 2; ++pp) {
                // word pp: K = 64Q + 16c + 8pp + [0, 8) -> four bf16x2 K pairs per row
                uint32_t f0[4], f1[4];
                dequant_word(pp ? w0.y : w0.x, s20, f0);
                dequant_word(pp ? w1.y : w1.x, s21, f1);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    // token 8nb + g, the same 8 K as the word
                    const uint4 b = lds128(sb + Q * C::kBQuarter + nb * 1024 + L.b[pp]);
                    mma_bf16_16816(acc[nb], f0[0], f1[0], f0[1], f1[1], b.x, b.y);
                    mma_bf16_16816(acc[nb], f0[2], f1[2], f0[3], f1[3], b.z, b.w);
                }
            }
        }
        // every shared-memory read of the stage has been consumed: hand it back
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[stage]);
        if (++stage == STAGES) { stage = 0; sphase ^= 1; }
    }
    return true;
}

template <int STAGES>
__global__ void __launch_bounds__(kWarpMmaThreads, 2)
grouped_gemm_int4_warp_kernel(const __grid_constant__ CUtensorMap tmA, const Params p) {
    using C = Int4WarpCfg<STAGES>;
    constexpr int BN = kWarpBN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ring = smem;                                    // STAGES x [A | B quarters 0..3]
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + C::kRingBytes);
    uint64_t *full_bar = bars;                               // producer (TMA bytes + 32 lanes' copies) -> MMA warps
    uint64_t *empty_bar = full_bar + STAGES;                 // MMA warps (8 arrivals) -> producer
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + C::kNumBars);
    int *off_s = reinterpret_cast<int *>(bars + C::kNumBars) + 16;   // [E+1]
    int *pre_s = off_s + (kMaxExperts + 1);                           // [E+1] tile prefix

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int E = p.E;
    const int MB = (p.m_out + C::kFeat - 1) / C::kFeat;
    const int KS = (p.K + 4 * kBK - 1) / (4 * kBK);          // stages of K = 256 per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1 + 32);                 // expect_tx arrival + one per producer lane
            mbar_init(&empty_bar[s], kWarpMmaWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) prefetch_tmap(&tmA);
    griddep_wait();
    build_tile_prefix<kWarpMmaThreads>(p.offsets, E, MB, BN, off_s, pre_s, p.P, p.err);
    __syncthreads();
    const int total_tiles = pre_s[E];

    if (warp == 0) {
        // ===================== producer: weights by TMA, tokens by cp.async =====
        const uint64_t pol_w = l2_policy_evict_first();     // weights are streamed once
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
            const int nrows = 8 * ((ti.valid + 7) >> 3);     // token rows the MMAs read
            // lane n holds the operand row of the tile's token row n; rows past
            // the tile's tokens are read but never stored, and rows past P
            // (the last expert's last block) read row 0
            const int my_r = ti.row0 + lane;
            const int my_row = (lane < nrows && my_r < p.P) ? token_row(p, my_r) : 0;
            const int a_row = ti.e * p.w_rows + ti.mb * C::kFeat;
            for (int ks = 0; ks < KS; ++ks) {
                if (lane == 0) ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.err, 256);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                uint8_t *st = ring + stage * C::kStageBytes;
                const uint32_t sb = smem_u32(st + C::kABytes);
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full_bar[stage], C::kABytes);
                    tma_load_2d(st, &tmA, &full_bar[stage], ks * 128, a_row, pol_w);
                }
                // lane L copies K = 256ks + 8L + [0, 8) of every token row: quarter
                // L / 8, 16-byte chunk L % 8, stored with the 128-byte swizzle
                const int kk = ks * 256 + 8 * lane;
                const uint32_t src_bytes = kk < p.K ? 16u : 0u;
                const uint32_t dq = sb + (lane >> 3) * C::kBQuarter;
                for (int n = 0; n < nrows; ++n) {
                    const int row = __shfl_sync(0xffffffffu, my_row, n);
                    const uint16_t *src = src_bytes ? p.a + static_cast<size_t>(row) * p.K + kk : p.a;
                    cp_async_16(dq + n * 128 + (((lane & 7) ^ (n & 7)) << 4), src, src_bytes);
                }
                cp_async_mbar_arrive_noinc(&full_bar[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else {
        // ============================ warps 1-8: decode + MMA ===================
        const int cw = warp - 1;
        const int g = lane >> 2, c = lane & 3;
        const int kgroups = p.K / 128;
        const size_t srows = static_cast<size_t>(p.E) * p.w_rows;
        // tile rows of MMA rows g (rr = 0) and g + 8 (rr = 1) of this warp
        const int brow[2] = {16 * cw + 2 * g, 16 * cw + 2 * g + 1};
        // chunk (2Q + c/2) ^ (r % 8) of row r = ((2Q) ^ (r % 8 & 6)) + ((c/2) ^ (r % 2))
        W4LaneOffsets L;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int r = brow[rr];
            L.a0[rr] = r * 128 + ((((c >> 1) ^ r) & 1) << 4) + 8 * (c & 1);
            L.ax[rr] = (r & 6) << 4;
        }
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) L.b[pp] = g * 128 + (((2 * c + pp) ^ g) << 4);
        int stage = 0;
        uint32_t sphase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
            const int nblk = (ti.valid + 7) >> 3;            // 8-token MMA blocks with a token in them
            // scale rows of MMA rows g, g + 8
            const size_t row0w = static_cast<size_t>(ti.e) * p.w_rows + ti.mb * C::kFeat;
            const size_t wr0 = row0w + brow[0];
            const size_t wr1 = row0w + brow[1];
            const bool s_ok = wr0 < srows && wr1 < srows;
            const uint16_t *sr0 = p.w_scales + wr0 * kgroups, *sr1 = p.w_scales + wr1 * kgroups;
            float acc[C::kNB][4];
#pragma unroll
            for (int nb = 0; nb < C::kNB; ++nb)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[nb][i] = 0.0f;
            if (nblk == 1)
                ok = mma_tile<STAGES, 1>(ring, full_bar, empty_bar, stage, sphase, KS, L, sr0, sr1, s_ok,
                                                 kgroups, abort_flag, p.err, acc);
            else if (nblk == 2)
                ok = mma_tile<STAGES, 2>(ring, full_bar, empty_bar, stage, sphase, KS, L, sr0, sr1, s_ok,
                                                 kgroups, abort_flag, p.err, acc);
            else if (nblk == 3)
                ok = mma_tile<STAGES, 3>(ring, full_bar, empty_bar, stage, sphase, KS, L, sr0, sr1, s_ok,
                                                 kgroups, abort_flag, p.err, acc);
            else
                ok = mma_tile<STAGES, 4>(ring, full_bar, empty_bar, stage, sphase, KS, L, sr0, sr1, s_ok,
                                                 kgroups, abort_flag, p.err, acc);
            if (!ok) break;

            // epilogue. C fragment of thread (g, c): acc[nb][h] is MMA row g and
            // acc[nb][2 + h] MMA row g + 8, for token 8nb + 2c + h.
#pragma unroll
            for (int nb = 0; nb < C::kNB; ++nb) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int t = 8 * nb + 2 * c + h;
                    if (nb < nblk && t < ti.valid) {
                        uint16_t *orow = p.out + static_cast<size_t>(ti.row0 + t) * p.m_out;
                        const int f0 = ti.mb * C::kFeat + brow[0];
                        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(acc[nb][h]));
                        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(acc[nb][2 + h]));
                        if (f0 + 1 < p.m_out) *reinterpret_cast<uint32_t *>(orow + f0) = lo | (hi << 16);
                    }
                }
            }
        }
    }

    // every role is done: the next kernel may start its set-up now
    griddep_launch_dependents();
    __syncthreads();
    if (*abort_flag) {
        // let the copies in flight land before the CTA exits
        for (int i = 0; i < 1000; ++i) __nanosleep(1000);
    }
}

template <int STAGES>
cudaError_t run_int4_warp(const GemmArgs &g, cudaStream_t s) {
    using C = Int4WarpCfg<STAGES>;
    CUtensorMap ta;
    const uint64_t a_rows = static_cast<uint64_t>(g.E) * g.w_rows;
    // packed weights: 128 bytes (K = 256) per row and stage, 128-byte swizzle
    if (!make_map(&ta, g.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, g.K / 2, a_rows, 128, C::kFeat,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    auto kern = grouped_gemm_int4_warp_kernel<STAGES>;
    cudaError_t st = ensure_dynamic_smem(kern, C::kSmemBytes);
    if (st != cudaSuccess) return st;
    const long long MB = (g.m_out + C::kFeat - 1) / C::kFeat;
    const long long max_tiles = ((static_cast<long long>(g.P) + kWarpBN - 1) / kWarpBN + std::min(g.E, g.P)) * MB;
    const int grid = static_cast<int>(std::min<long long>(2LL * num_sms(), max_tiles));
    if (grid <= 0) return cudaSuccess;
    return launch_pdl(kern, dim3(grid), dim3(kWarpMmaThreads), C::kSmemBytes, s, ta, make_params(g, kWarpBN));
}

}  // namespace

cudaError_t launch_grouped_gemm_int4_warp(const GemmArgs &g, cudaStream_t s) {
    if (g.swiglu || g.fmt != 1) return cudaErrorInvalidValue;   // the int4 down GEMM only
    return run_int4_warp<3>(g, s);
}

}  // namespace moe
