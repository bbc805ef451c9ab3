// gemm_decode.cuh -- the W8A8 / W4A8 GEMM for few tokens (M <= 64; int8
// weights also up to 128 tokens where the one-CTA kernel's tiles would leave
// most SMs idle), included by gemm.cu (it shares that file's PTX wrappers
// and fault word).
//
// Same operation as w8a8_gemm_kernel: y = dequant(qx qw^T) (CUDA INT8
// quantization notes, aicoding.csdn.net, sections 3.2 and 4.2).  With few
// tokens the product is bound by the weight bytes, and a 128 x 256 tile per
// CTA leaves most of the tensor-core tile empty and only N/256 CTAs to
// stream the weights.  Here the operands swap roles:
//
//   * the MMA's A operand (M = 128, TMEM lanes) is a 128-row weight tile,
//     its B operand (N = NT = 16, 32, 64 or 128) the token tile; D[n][t] lands
//     in TMEM lane n, column t, so the epilogue thread of weight row n
//     writes y[t][n] for every token (32 lanes = 32 consecutive columns of
//     y: coalesced);
//   * one CTA per 128 weight rows, about 108 KB of shared memory so that two
//     CTAs share an SM, every CTA resident at once: the weight stream is
//     spread over all SMs and HBM shares itself among the CTAs;
//   * where N / 128 tiles are too few to fill the SMs, the K dimension is
//     split over a thread-block cluster of S CTAs (S <= 8): each CTA
//     accumulates its share of the k-blocks, writes the int32 partial to
//     its shared memory, and after a cluster barrier CTA rank r sums the
//     S partials of rows [r 128/S, (r+1) 128/S) through distributed shared
//     memory (exact int32) and runs the dequant for them.  No global
//     scratch memory;
//   * int4 weights (two per byte) arrive packed, 256 K a k-block (128-byte
//     rows, TMA 128B swizzle), and are unpacked by eight converter warps
//     straight into tensor memory, which the MMA reads as its A operand
//     (three unpacked tiles in flight); the first four converter warps
//     then run the epilogue.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps
// 2..5 epilogue (int4: warps 2..9 convert first, in two groups of four).  Every wait is bounded as in the
// other GEMM kernels; no TMA multicast.

namespace w8a8 {
namespace gemm {

#ifndef W8A8_DEC_OP_STAGES
#define W8A8_DEC_OP_STAGES 3
#endif
#ifndef W8A8_DEC_CONV_WARPS
#define W8A8_DEC_CONV_WARPS 8
#endif
#ifndef W8A8_DEC_CONV_GROUPS
#define W8A8_DEC_CONV_GROUPS 2
#endif
constexpr int kDecRows = 128;  // weight rows per CTA (= MMA M = TMEM lanes)
constexpr int kDecConvWarps = W8A8_DEC_CONV_WARPS;  // int4 unpacking warps (the first 4 also run the epilogue)
// the converter warps form groups of four (one warp per TMEM lane quarter,
// one weight row per thread) that take alternate k-blocks, so that several
// stages are unpacked at once (the unpacking of one stage is latency-bound:
// shared loads, ALU, TMEM store, fence, arrive)
constexpr int kDecConvGroups = W8A8_DEC_CONV_GROUPS;
constexpr int kDecConvGroupThreads = kDecConvWarps * 32 / kDecConvGroups;
// producer, MMA, then 4 epilogue warps (int4: the converter warps)
__host__ __device__ constexpr int dec_threads(bool int4) { return 64 + 32 * (int4 ? kDecConvWarps : 4); }
constexpr int kDecMaxSplit = 8;   // portable cluster size
constexpr int kDecMaxTokens = 64;
constexpr int kDecBudget = 108 * 1024;  // dynamic shared memory, two CTAs per SM

// K per k-block: int4 weights take 256 (128 packed bytes a row, as many
// bytes a stage as int8's 128), which halves the k-blocks and so the
// per-k-block handshakes of the unpacking pipeline
__host__ __device__ constexpr int dec_kblock(bool int4) { return int4 ? 2 * BK : BK; }

template <int NT, bool INT4>
struct CfgDec {
    static constexpr int KB = dec_kblock(INT4);
    static constexpr int W_BYTES = kDecRows * BK;                         // int8 weight tile (MMA A)
    static constexpr int RAW_BYTES = INT4 ? kDecRows * KB / 2 : W_BYTES;  // weight tile as loaded
    static constexpr int X_ATOM = NT * BK;                                // token rows x 128 bytes (one swizzle atom)
    static constexpr int X_BYTES = NT * KB;                               // token tile (MMA B), KB / 128 atoms
    static constexpr int IN_BYTES = RAW_BYTES + X_BYTES;
    static constexpr int OP_STAGES = INT4 ? W8A8_DEC_OP_STAGES : 0;  // unpacked weight tiles (in TMEM)
    static constexpr int IN_OFFSET = 0;
    static constexpr int STAGES_FIT = (kDecBudget - IN_OFFSET) / IN_BYTES;
    static constexpr int STAGES = STAGES_FIT < 8 ? STAGES_FIT : 8;
    static constexpr int SMEM = IN_OFFSET + STAGES * IN_BYTES + 1024;  // + alignment slack
    // TMEM: the accumulator (NT columns), then OP_STAGES unpacked weight
    // tiles of KB / 4 columns (128 rows x KB int8, four per 32-bit column)
    static constexpr int ACC_COLS = NT < 32 ? 32 : NT;
    static constexpr int A_COLS = KB / 4;
    static constexpr int USED_COLS = ACC_COLS + OP_STAGES * A_COLS;
    static constexpr int TMEM_COLS = USED_COLS <= 32 ? 32 : USED_COLS <= 64 ? 64 : USED_COLS <= 128 ? 128 : 256;
    static_assert(USED_COLS <= 256, "two CTAs per SM share 512 TMEM columns");
    static constexpr int RED_BYTES = NT * kDecRows * 4;  // int32 partial, over the stages
    static_assert(STAGES >= 3, "decode pipeline too shallow");
    // a converter group's previous k-block (kb - G) made it wait for the MMA
    // to consume kb - G - OP_STAGES, so every barrier it waits on next is at
    // most one phase behind (an mbarrier parity wait cannot tell two phases
    // apart): G <= OP_STAGES
    static_assert(!INT4 || (kDecConvGroups >= 1 && kDecConvGroups <= OP_STAGES && STAGES >= OP_STAGES),
                  "converter groups must not run more than one phase ahead");
    static_assert(!INT4 || kDecConvGroupThreads == kDecRows, "a converter group is one thread per weight row");
    static_assert(IN_BYTES % 1024 == 0 && RAW_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");
    static_assert(RED_BYTES <= STAGES * IN_BYTES, "partial must fit over the stages");
};

__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t map_to_rank(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}

__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// y[t][n] (and acc_out[t][n]) from the full accumulator of weight row n and
// token t.
template <typename OutT, bool ASYM>
__device__ __forceinline__ void dec_store(int32_t acc, int t, int n, int N, const float *__restrict__ sx,
                                          const int32_t *__restrict__ rs, float swv, float owv,
                                          OutT *__restrict__ y, int32_t *__restrict__ acc_out) {
    const float v = dequant1<ASYM>((uint32_t)acc, sx[t], ASYM ? rs[t] : 0, swv, owv);
    const int64_t at = (int64_t)t * N + n;
    if (sizeof(OutT) == 2)
        reinterpret_cast<__nv_bfloat16 *>(y)[at] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float *>(y)[at] = v;
    if (acc_out) acc_out[at] = acc;
}

// Synchronisation:
//   in_full[s]  : producer's expect_tx; the weight and token TMAs complete it.
//   in_empty[s] : MMA commit (the MMA is the last reader of a stage).
//   op_full[p]  : int4: one arrival per converter thread after its TMEM
//                 stores completed and were fenced (it waited for in_full
//                 first, so op_full implies it).
//   op_empty[p] : int4: MMA commit (the MMA is the last reader of the
//                 unpacked tile in TMEM).
//   tfull       : MMA commit after the CTA's last k-block.
template <int NT, typename OutT, bool ASYM, bool INT4>
__global__ void __launch_bounds__(dec_threads(INT4), 2)
w8a8_gemm_decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                        const float *__restrict__ sx, const float *__restrict__ sw,
                        const int32_t *__restrict__ rs, const float *__restrict__ ow, OutT *__restrict__ y,
                        int32_t *__restrict__ acc_out, int M, int N, int K) {
    using C = CfgDec<NT, INT4>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t in_full[C::STAGES];
    __shared__ __align__(8) uint64_t in_empty[C::STAGES];
    __shared__ __align__(8) uint64_t op_full[INT4 ? C::OP_STAGES : 1];
    __shared__ __align__(8) uint64_t op_empty[INT4 ? C::OP_STAGES : 1];
    __shared__ __align__(8) uint64_t tfull_bar;
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;  // 1024-aligned for 128B swizzle
    uint8_t *gbase = smem_raw + (smem_base - smem_u32(smem_raw));      // the same bytes, generic address

    // K split over the cluster (1 CTA, rank 0, without a cluster launch)
    const int split = (int)cluster_nctarank();
    const int rank = (int)cluster_ctarank();
    const int n0 = (int)(blockIdx.x / split) * kDecRows;
    const int num_kb = (K + C::KB - 1) / C::KB;
    const int kb0 = (int)((int64_t)num_kb * rank / split);
    const int kb1 = (int)((int64_t)num_kb * (rank + 1) / split);  // the host keeps kb1 > kb0

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(smem_u32(&in_full[s]), 1);
            mbar_init(smem_u32(&in_empty[s]), 1);
        }
        for (int p = 0; p < C::OP_STAGES; ++p) {
            mbar_init(smem_u32(&op_full[p]), kDecConvGroupThreads);  // one group unpacks a stage
            mbar_init(smem_u32(&op_empty[p]), 1);
        }
        mbar_init(smem_u32(&tfull_bar), 1);
        mbar_init(smem_u32(&drain_bar), 1);
        abort_flag = 0;
        fence_barrier_init();
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmap_w) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmap_x) : "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    pdl_wait();     // the codes and scales come from the previous kernel (prologue above overlapped it)
    pdl_trigger();  // the next kernel may launch; it waits for this grid before touching memory

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!wait_bounded(smem_u32(&in_empty[stage]), phase ^ 1u, &abort_flag, kFaultProducer)) {
                    ok = false;
                    break;
                }
                const uint32_t w_dst = smem_base + C::IN_OFFSET + stage * C::IN_BYTES;
                const uint32_t fb = smem_u32(&in_full[stage]);
                // token atoms that start inside K (the weights' tail is zero-filled)
                const int atoms = min(C::KB / BK, (K - kb * C::KB + BK - 1) / BK);
                mbar_arrive_expect_tx(fb, C::RAW_BYTES + atoms * C::X_ATOM);
                tma_load_2d(w_dst, &tmap_w, fb, INT4 ? kb * (C::KB / 2) : kb * BK, n0);
                for (int a = 0; a < atoms; ++a)
                    tma_load_2d(w_dst + C::RAW_BYTES + a * C::X_ATOM, &tmap_x, fb, kb * C::KB + a * BK, 0);
                ++issued;
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                // drain: wait (bounded) for the copies of the last issued stages
                int outstanding = issued < C::STAGES ? issued : C::STAGES;
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < outstanding; ++i) {
                    if (--s < 0) {
                        s = C::STAGES - 1;
                        ph ^= 1u;
                    }
                    const unsigned long long t0 = globaltimer();
                    while (!mbar_try_wait(smem_u32(&in_full[s]), ph) && globaltimer() - t0 < kWaitNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kDecRows, NT);
            int stage = 0, os = 0;
            uint32_t phase = 0, oph = 0;
            bool ok = true, issued_any = false;
            for (int kb = kb0; kb < kb1; ++kb) {
                const uint32_t bar = INT4 ? smem_u32(&op_full[os]) : smem_u32(&in_full[stage]);
                if (!wait_bounded(bar, INT4 ? oph : phase, &abort_flag, kFaultMmaFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t in_addr = smem_base + C::IN_OFFSET + stage * C::IN_BYTES;
                const uint32_t b_addr = in_addr + C::RAW_BYTES;
                // MMA steps that start inside K (K is a multiple of 16, and of 32 for int4)
                const int steps = min(C::KB / UMMA_K, (K - kb * C::KB + UMMA_K - 1) / UMMA_K);
#pragma unroll
                for (int k = 0; k < C::KB / UMMA_K; ++k) {
                    if (k >= steps) break;
                    const uint32_t acc = (kb > kb0 || k > 0) ? 1u : 0u;
                    // B: token atom k / 4, 32 bytes per step within its 128-byte rows
                    const uint32_t bk = b_addr + (uint32_t)((k / (BK / UMMA_K)) * C::X_ATOM + (k % (BK / UMMA_K)) * UMMA_K);
                    if (INT4)  // A: the unpacked tile in TMEM, UMMA_K / 4 columns per step
                        mma_i8_tmem_a(tmem_base, tmem_base + (uint32_t)(C::ACC_COLS + os * C::A_COLS + k * (UMMA_K / 4)),
                                      smem_desc_sw128(bk), idesc, acc);
                    else
                        mma_i8(tmem_base, smem_desc_sw128(in_addr + k * UMMA_K), smem_desc_sw128(bk), idesc, acc);
                }
                issued_any = true;
                mma_commit(smem_u32(&in_empty[stage]));
                if (INT4) mma_commit(smem_u32(&op_empty[os]));
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
                if (++os == C::OP_STAGES) {
                    os = 0;
                    oph ^= 1u;
                }
            }
            if (ok) {
                mma_commit(smem_u32(&tfull_bar));
            } else if (issued_any) {
                // drain: every MMA issued so far completes before TMEM is freed
                mma_commit(smem_u32(&drain_bar));
                const unsigned long long t0 = globaltimer();
                while (!mbar_try_wait(smem_u32(&drain_bar), 0) && globaltimer() - t0 < kWaitNs) {
                }
            }
        }
    } else {
        const int ct = threadIdx.x - 64;
        bool ok = true;
        if (INT4) {
            // ------------------------------------------ converters
            // A packed tile is 128 rows x 128 bytes (TMA 128B swizzle:
            // piece j of row r at piece j ^ (r & 7), so the 8 rows a
            // quarter-warp reads at once fall in distinct banks).  Each
            // thread unpacks one weight row r = 32 (warp % 4) + lane (a
            // warp may only access TMEM lanes 32 (warp % 4) ..), 256 codes,
            // into 64 words, stored in two halves to lane r, columns
            // [ACC_COLS + 64 p, +64) for unpacked tile p.  Group g takes the
            // k-blocks kb0 + g, kb0 + g + G, ...; the ring positions and
            // phases follow from the k-block's index.
            constexpr int kOps = INT4 ? C::OP_STAGES : 1;  // (this branch only runs for int4)
            const int grp = ct / kDecConvGroupThreads;
            const int row = (warp & 3) * 32 + lane;  // this thread's TMEM lane = weight row of the tile
            const uint32_t lane_base = tmem_base + ((uint32_t)((warp & 3) * 32) << 16);
            const int rot = row & 7;
            for (int kb = kb0 + grp; kb < kb1; kb += kDecConvGroups) {
                const int u = kb - kb0;
                const int stage = u % C::STAGES, os = u % kOps;
                const uint32_t phase = (uint32_t)(u / C::STAGES) & 1u, oph = (uint32_t)(u / kOps) & 1u;
                const bool got = wait_bounded(smem_u32(&op_empty[os]), oph ^ 1u, &abort_flag, kFaultConvert) &&
                                 wait_bounded(smem_u32(&in_full[stage]), phase, &abort_flag, kFaultConvert);
                if (!__all_sync(0xffffffffu, got)) {  // the TMEM store below is warp-collective
                    ok = false;
                    break;
                }
                tc_fence_after();  // the MMA that last read this tile is done
                const uint8_t *rowp = gbase + C::IN_OFFSET + stage * C::IN_BYTES + row * (C::KB / 2);
#pragma unroll
                for (int h = 0; h < C::KB / 128; ++h) {
                    uint32_t o[32];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint4 p = *reinterpret_cast<const uint4 *>(rowp + (((4 * h + j) ^ rot) << 4));
                        unpack_int4x8(p.x, o[8 * j + 0], o[8 * j + 1]);
                        unpack_int4x8(p.y, o[8 * j + 2], o[8 * j + 3]);
                        unpack_int4x8(p.z, o[8 * j + 4], o[8 * j + 5]);
                        unpack_int4x8(p.w, o[8 * j + 6], o[8 * j + 7]);
                    }
                    tmem_st32(lane_base + (uint32_t)(C::ACC_COLS + os * C::A_COLS + 32 * h), o);
                }
                tc_fence_before();  // the stores are ordered before the arrive the MMA waits on
                mbar_arrive(smem_u32(&op_full[os]));
            }
        }
        // ---------------------------------------------- epilogue (warps 2..5)
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int nl = quarter * 32 + lane;
        const int n = n0 + nl;
        if (ok && warp < 6) ok = wait_bounded(smem_u32(&tfull_bar), 0, &abort_flag, kFaultEpilogue);
        // the TMEM loads below are warp-collective: all lanes or none
        // (warps 6.. only convert)
        if (warp < 6 && __all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            const float swv = n < N ? sw[n] : 0.0f;
            const float owv = (ASYM && n < N) ? ow[n] : 0.0f;
            int32_t *red = reinterpret_cast<int32_t *>(gbase + C::IN_OFFSET);
#pragma unroll
            for (int c0 = 0; c0 < NT; c0 += 16) {
                uint32_t acc[16];
                tmem_ld16(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0, acc);
                if (INT4) {  // 16 times the product (see unpack_int4x8); exact
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[j] = (uint32_t)((int32_t)acc[j] >> kInt4AccShift);
                }
                if (split == 1) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c0 + j < M && n < N)
                            dec_store<OutT, ASYM>((int32_t)acc[j], c0 + j, n, N, sx, rs, swv, owv, y, acc_out);
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) red[(c0 + j) * kDecRows + nl] = (int32_t)acc[j];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (split > 1) {
        // every CTA of the cluster holds its partial in shared memory: rank r
        // sums rows [r R, (r + 1) R) of all S partials, R = 128 / S
        cluster_sync_all();
        const int rows = kDecRows / split;
        const uint32_t red_base = smem_base + C::IN_OFFSET;
        for (int e = threadIdx.x; e < NT * rows; e += (int)blockDim.x) {
            const int t = e / rows, nl = rank * rows + e % rows;
            const int n = n0 + nl;
            if (t < M && n < N) {
                const uint32_t local = red_base + (uint32_t)((t * kDecRows + nl) * 4);
                int32_t sum = 0;
                for (int p = 0; p < split; ++p) sum += ld_cluster_s32(map_to_rank(local, (uint32_t)p));
                dec_store<OutT, ASYM>(sum, t, n, N, sx, rs, sw[n], ASYM ? ow[n] : 0.0f, y, acc_out);
            }
        }
        cluster_sync_all();  // no CTA leaves while a peer still reads its partial
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace gemm
}  // namespace w8a8
