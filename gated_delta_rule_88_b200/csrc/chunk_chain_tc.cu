// chunk_chain_tc.cu -- the sequential inter-chunk pass of the bf16 KDA prefill
// on the Blackwell tensor cores (tcgen05 MMAs, accumulators in TMEM, records
// streamed by bulk async copies).  dk = dv = 128, C = 64.
//
// Kimi Linear paper notes (paper-notes-site), section 3: only the fixed-size
// state passes between chunks; the output is the inter-chunk part plus the
// intra-chunk part.  With the per-chunk record of chunk_ws.h, for each chunk in
// order and one DVT-column tile of the fp32 state S (dk x DVT):
//     MMA1  D1 = [W; Qg] S            (M = 128: rows 0-63 W S, 64-127 Qg S)
//           V_new = U - (W S)         (threads 0-63, one token row each)
//     MMA2  D1 += [* ; P] V_new       (rows 64-127 become O = Qg S + P V_new)
//     MMA3  D3 = Kt^T V_new           (M = 128 channels)
//           S <- Diag(e^{G_C}) S + D3 (threads 0-127, one channel row each)
// The state stays in fp32 registers for the whole sequence; its bf16 copy is
// the B operand of MMA1.  A operands come straight from the record (K-major,
// 128-byte swizzle); B operands (S, V_new) are written by the threads as
// MN-major operands swizzled to the tile width (rows of 32 to 128 bytes).
//
// Roles (192 threads): warps 0-3 are the epilogue (thread t <-> TMEM lane t:
// token row t of D1, channel row t of D3); warp 4 lane 0 streams records into
// an NS-stage shared-memory ring with cp.async.bulk (plain, no multicast) and
// mbarrier transaction counts; warp 5 lane 0 issues the MMAs.  The issuer and
// the epilogue meet at two OR-reduced named barriers per chunk (S ready, V_new
// ready), which also carry failures, so every party leaves the loop at the
// same barrier.  Every wait is bounded: a wait that runs out sets the device
// error word; the CTA then drains its copies and MMAs (bounded), frees TMEM and
// returns.
#include "chunk_ws.h"
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = ws::C;
constexpr int D = ws::D;
constexpr uint32_t REC_HEAD = 57344;       // [W;Qg] + Kt^T + P, contiguous in the record

template <int DVT, int NS>
struct TcLayout {
    // epilogue: one warp per (TMEM lane quarter, group of CPT columns)
    static constexpr int CPT = DVT < 32 ? DVT : 32;          // columns per epilogue thread
    static constexpr int CGRP = DVT / CPT;                   // column groups
    static constexpr int EPI = 4 * CGRP;                     // epilogue warps
    static constexpr int NTHREADS = 32 * (EPI + 3);          // + loader + two MMA issuers
    static constexpr int UT = DVT > 32 ? DVT / 32 : 1;
    static constexpr uint32_t U_OFF = REC_HEAD;
    static constexpr uint32_t EGC_OFF = REC_HEAD + UT * 4096;
    static constexpr uint32_t STAGE = ((EGC_OFF + 512 + 1023) / 1024) * 1024;
    static constexpr uint32_t TX = REC_HEAD + UT * 4096 + 512;
    static constexpr uint32_t B1_OFF = NS * STAGE;                 // S^bf16: K=128 x N=DVT
    static constexpr uint32_t B2_OFF = B1_OFF + 128 * DVT * 2;     // V_new: K=64 x N=DVT, two buffers
    static constexpr uint32_t B2_BYTES = 64 * DVT * 2;
    static constexpr uint32_t BAR_OFF = B2_OFF + 2 * B2_BYTES;
    static constexpr uint32_t BYTES = BAR_OFF + 8 * (2 * NS + 8) + 16;
    // TMEM columns: D1 double-buffered (2 x DVT) + D3 (DVT), rounded to a power of 2
    static constexpr uint32_t NCOLS = 3 * DVT <= 32 ? 32 : 3 * DVT <= 64 ? 64 : 3 * DVT <= 128 ? 128
                                    : 3 * DVT <= 256 ? 256 : 512;
    // B operands S and V_new: MN-major, swizzled to the tile width (rows of
    // DVT bf16 = 32, 64 or 128 bytes; at DVT = 128 two 64-column atoms of
    // 128-byte rows, the second B1_ATOM / B2_ATOM bytes after the first),
    // 8-row groups contiguous
    static constexpr int NATOM = DVT > 64 ? DVT / 64 : 1;
    static constexpr uint32_t BW = DVT > 64 ? 128 : DVT * 2;
    static constexpr uint32_t B_SBO = 8 * BW;
    static constexpr uint32_t B1_ATOM = 128 * BW;                  // K = 128 channel rows
    static constexpr uint32_t B2_ATOM = 64 * BW;                   // K = 64 token rows
    static constexpr uint32_t B1_LBO = NATOM > 1 ? B1_ATOM : B_SBO;
    static constexpr uint32_t B2_LBO = NATOM > 1 ? B2_ATOM : B_SBO;
    static constexpr uint32_t B_LAYOUT = DVT >= 64 ? 2 : DVT == 32 ? 4 : 6;   // 128 / 64 / 32-byte swizzle
    static constexpr int B_SWZ = DVT >= 64 ? 7 : DVT == 32 ? 3 : 1;
    // byte offset of the 16-byte chunk `chunk` (8 columns) of K row k, in an
    // operand whose 64-column atoms are ATOM bytes apart
    template <uint32_t ATOM>
    static __device__ __forceinline__ uint32_t b_off(int k, int chunk) {
        const uint32_t a = NATOM > 1 ? (uint32_t)(chunk >> 3) * ATOM : 0u;
        const int j = NATOM > 1 ? (chunk & 7) : chunk;
        return a + (k >> 3) * B_SBO + (k & 7) * BW + ((j ^ ((((k & 7) * BW) >> 7) & B_SWZ)) << 4);
    }
};

template <int DVT, int NS>
__global__ void __launch_bounds__(TcLayout<DVT, NS>::NTHREADS, 1)
chunk_chain_tc_kernel(const unsigned char *__restrict__ wsp, const int32_t *__restrict__ cu,
                      const int32_t *__restrict__ coff, const float *__restrict__ s0,
                      float *__restrict__ sT, __nv_bfloat16 *__restrict__ out, int T, int total_T,
                      int H, int cps, int max_chunks, int *__restrict__ err,
                      unsigned char *__restrict__ s_img, unsigned char *__restrict__ v_img,
                      const int32_t *__restrict__ order, int out_v8)
{
    using L = TcLayout<DVT, NS>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::BAR_OFF);
    uint64_t *empty = full + NS;
    uint64_t *mma1 = empty + NS;
    uint64_t *mma3 = mma1 + 1;
    uint64_t *mma2 = mma1 + 2;                         // [2]: MMA2(i) done, by i & 1
    uint64_t *drain = mma1 + 4;                        // [2]: one per issuer
    uint64_t *s_go = mma1 + 6;                         // [2]: MMA3(i) issued, by i & 1
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma1 + 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    unsigned char *B1 = sm + L::B1_OFF;
    unsigned char *B2 = sm + L::B2_OFF;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // varlen: sequences longest first (order from chunk_plan_kernel), so the
    // longest chains start in the first wave
    const int n0 = blockIdx.x * DVT, h = blockIdx.y;
    const int seq = order ? order[blockIdx.z] : blockIdx.z;

    long long bos, eos;
    int c_begin;
    if (cu) {
        bos = min(max(cu[seq], 0), total_T);
        eos = min(max(cu[seq + 1], 0), total_T);
        if (eos < bos) eos = bos;
        c_begin = coff[seq];
    } else {
        bos = (long long)seq * T;
        eos = bos + T;
        c_begin = seq * cps;
    }
    int nchunks = (int)((eos - bos + C - 1) / C);
    if (c_begin < 0 || c_begin + nchunks > max_chunks) {
        if (tid == 0) set_device_error(err, kErrBadOffsets);
        nchunks = c_begin < 0 ? 0 : max(0, min(nchunks, max_chunks - c_begin));
    }
    const unsigned char *rec0 = wsp + ((size_t)max(c_begin, 0) * H + h) * ws::RECORD;
    const size_t rec_stride = (size_t)H * ws::RECORD;

    if (tid == 0) {
        // a stage is free once both issuers' MMAs on it are done
        for (int s = 0; s < NS; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 2); }
        mbar_init(mma1, 1);
        mbar_init(mma3, 1);
        for (int b = 0; b < 2; ++b) { mbar_init(&mma2[b], 1); mbar_init(&drain[b], 1); mbar_init(&s_go[b], 1); }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(tmem_slot, L::NCOLS); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr int BAR_S = 1, BAR_V = 2, BAR_O = 3;     // named barriers (0 = __syncthreads)
    constexpr int EPI = L::EPI, CPT = L::CPT;
    constexpr int NSYNC = 32 * EPI + 32;               // epilogue warps + the chain issuer warp
    constexpr int NOUT = 32 * EPI / 2;                 // epilogue threads on TMEM lanes 64-127

    if (warp == EPI) {
        // ---------------- loader ----------------
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < nchunks; ++i) {
                const int s = i % NS;
                if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) {
                    set_device_error(err, kErrWaitTimeout);
                    break;
                }
                if (*abort_flag) break;
                const unsigned char *rec = rec0 + (size_t)i * rec_stride;
                unsigned char *st = sm + (size_t)s * L::STAGE;
                mbar_arrive_expect_tx(&full[s], L::TX);
                bulk_g2s(st, rec, REC_HEAD, &full[s]);
                bulk_g2s(st + L::U_OFF, rec + ws::OFF_U + (size_t)(n0 >> 5) * ws::U_TILE,
                         L::UT * 4096, &full[s]);
                bulk_g2s(st + L::EGC_OFF, rec + ws::OFF_EGC, 512, &full[s]);
                if (i + NS < nchunks) bulk_prefetch_l2(rec + (size_t)NS * rec_stride, ws::RECORD);
                issued = i + 1;
            }
            // never leave with copies in flight into this CTA's shared memory
            for (int j = max(0, issued - NS); j < issued; ++j)
                mbar_wait(&full[j % NS], (j / NS) & 1, 1u << 20);
        }
    } else if (warp == EPI + 1 || warp == EPI + 2) {
        // ---------------- MMA issuers: warp EPI + 1 lane 0 the chain (MMA1, MMA3;
        // the warp joins the barriers), warp EPI + 2 lane 0 the output product (MMA2) ----------------
        constexpr uint32_t IDESC = idesc_bf16(128, DVT, true);
        // A operands: K-major, 128-byte swizzle, 8-row groups 1024 B apart, relative
        // to the ring base; B operands: MN-major, swizzled to the tile width
        const uint32_t sm_a = smem_u32(sm);
        const DescParts a_sw = smem_desc_parts(sm_a, 16, 1024, 2);
        const DescParts b1_d = smem_desc_parts(smem_u32(B1), L::B1_LBO, L::B_SBO, L::B_LAYOUT);
        const DescParts b2_d0 = smem_desc_parts(smem_u32(B2), L::B2_LBO, L::B_SBO, L::B_LAYOUT);
        const DescParts b2_d1 = smem_desc_parts(smem_u32(B2 + L::B2_BYTES), L::B2_LBO, L::B_SBO, L::B_LAYOUT);
        constexpr uint32_t BK = (2 * L::B_SBO) >> 4;       // descriptor step per 16 K rows
        bool issued_any = false;
        if (warp == EPI + 1) for (int i = 0; i < nchunks; ++i) {
            const int s = i % NS;
            const int p = i & 1;
            const uint32_t a_lo = a_sw.lo + ((uint32_t)s * L::STAGE >> 4);
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&full[s], (i / NS) & 1);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (named_bar_or(BAR_S, NSYNC, !ok)) break;        // S_i is in B1
            tc_fence_after();
            if (lane == 0) {
                const uint32_t d1 = tmem + p * DVT;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16_p(d1, a_lo + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), a_sw.hi,
                                b1_d.lo + (kk * BK), b1_d.hi, IDESC, kk > 0);
                umma_commit(mma1);
                issued_any = true;
            }
            __syncwarp();
            if (named_bar_or(BAR_V, NSYNC, false)) break;      // V_new is in B2[p]
            tc_fence_after();
            if (lane == 0) {
                // the state update (MMA3) is the sequential path; the output
                // product (MMA2) goes to the second issuer
                const uint32_t b2_lo = p ? b2_d1.lo : b2_d0.lo;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16_p(tmem + 2 * DVT, a_lo + (((uint32_t)ws::OFF_KTT + kk * 32) >> 4),
                                a_sw.hi, b2_lo + (kk * BK), b2_d0.hi, IDESC, kk > 0);
                umma_commit(mma3);
                umma_commit(&empty[s]);
                mbar_arrive(&s_go[p]);
            }
            __syncwarp();
        }
        if (warp == EPI + 2 && lane == 0) for (int i = 0; i < nchunks; ++i) {
            // MMA2: O rows (64-127 of D1[p]) += P V_new, once MMA3(i) is issued.
            // s_go[p] cannot run two phases ahead: MMA3(i + 2) needs the
            // epilogue past emit(i) (after BAR_V(i + 1)), which waits for
            // this MMA2.
            const int s = i % NS;
            const int p = i & 1;
            bool ok = false;
            for (uint32_t it = 0; it < (1u << 24); ++it) {
                if (mbar_test_wait(&s_go[p], (i >> 1) & 1)) { ok = true; break; }
                if (*abort_flag) break;
                if (it > 64) __nanosleep(32);
            }
            if (!ok) { set_device_error(err, kErrWaitTimeout); break; }
            tc_fence_after();
            const uint32_t a_lo = a_sw.lo + ((uint32_t)s * L::STAGE >> 4);
            const uint32_t b2_lo = p ? b2_d1.lo : b2_d0.lo;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16_p(tmem + p * DVT, a_lo + (((uint32_t)ws::OFF_P - 8192 + kk * 32) >> 4),
                            a_sw.hi, b2_lo + (kk * BK), b2_d0.hi, IDESC, 1);
            umma_commit(&mma2[p]);
            umma_commit(&empty[s]);
            issued_any = true;
        }
        // never free TMEM under a running MMA
        if (lane == 0 && issued_any) {
            umma_commit(&drain[warp - EPI - 1]);
            mbar_wait(&drain[warp - EPI - 1], 0, 1u << 20);
        }
    } else {
        // ---------------- epilogue warps 0 .. EPI-1: thread <-> TMEM lane t =
        // 32 (warp % 4) + lane (token row t of D1, channel row t of D3), columns
        // cb .. cb + CPT - 1 of the tile with cb = CPT (warp / 4) ----------------
        const int t = 32 * (warp & 3) + lane;
        const int cb = CPT * (warp >> 2);
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        float S[CPT];
        {
            const size_t sb = (((size_t)seq * H + h) * D + t) * D + n0 + cb;
#pragma unroll
            for (int j = 0; j < CPT; j += 4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (s0) x = *reinterpret_cast<const float4 *>(s0 + sb + j);
                S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
            }
        }
        // S entering chunk ci -> B1; with s_img (the backward's forward pass)
        // also its bf16 image [dk][dv], K-major SW128 in 64-column blocks
        auto write_B1 = [&](int ci) {
            unsigned char *img = (s_img && ci < nchunks)
                                     ? s_img + ((size_t)(max(c_begin, 0) + ci) * H + h) * 32768 : nullptr;
#pragma unroll
            for (int ng = 0; ng < CPT / 8; ++ng) {
                uint4 pk = make_uint4(pack_bf16(S[8 * ng], S[8 * ng + 1]), pack_bf16(S[8 * ng + 2], S[8 * ng + 3]),
                                      pack_bf16(S[8 * ng + 4], S[8 * ng + 5]), pack_bf16(S[8 * ng + 6], S[8 * ng + 7]));
                *reinterpret_cast<uint4 *>(B1 + L::template b_off<L::B1_ATOM>(t, cb / 8 + ng)) = pk;
                if (img) {
                    const int n = n0 + cb + 8 * ng;
                    *reinterpret_cast<uint4 *>(img + (size_t)(n >> 6) * 16384 + ws::sw128(t, n & 63)) = pk;
                }
            }
            fence_proxy_async_smem();
        };
        // CPT columns of lane t starting at tile column col + cb
        auto tmem_row = [&](uint32_t col, float (&x)[CPT]) {
            if constexpr (CPT == 16) {
                tmem_ld16(tmem + lane_base + col + cb, x);
            } else {
                tmem_ld32(tmem + lane_base + col + cb, x);
            }
            tmem_wait_ld();
        };
        // O of chunk ci (rows 64-127 of D1[ci & 1]) -> out; the warps on TMEM
        // lanes 64-127 only, between BAR_S and BAR_V of chunk ci + 1.  One
        // barrier per D1 buffer: MMA2(ci + 2) needs BAR_V(ci + 2), which needs
        // this call, so each wait is at most one phase behind.
        auto emit_output = [&](int ci) -> bool {
            bool okk = true;
            if (t == 64 && cb == 0) okk = mbar_wait(&mma2[ci & 1], (ci >> 1) & 1);
            if (named_bar_or(BAR_O, NOUT, !okk)) return false;
            tc_fence_after();
            const long long tok = bos + (long long)C * ci + (t - 64);
            float o[CPT];
            tmem_row((ci & 1) * DVT, o);
            if (out && tok < eos) {        // out == nullptr: the backward's recompute pass
                __nv_bfloat16 *row = out + ((size_t)tok * H + h) * D + n0 + cb;
                if (out_v8) {
                    // 16 columns = one 32-byte sector per store
#pragma unroll
                    for (int e = 0; e < CPT / 16; ++e) {
                        const float *x = o + 16 * e;
                        asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"l"(row + 16 * e),
                                     "r"(pack_bf16(x[0], x[1])), "r"(pack_bf16(x[2], x[3])), "r"(pack_bf16(x[4], x[5])),
                                     "r"(pack_bf16(x[6], x[7])), "r"(pack_bf16(x[8], x[9])), "r"(pack_bf16(x[10], x[11])),
                                     "r"(pack_bf16(x[12], x[13])), "r"(pack_bf16(x[14], x[15]))
                                     : "memory");
                    }
                } else {
                    uint4 *dst = reinterpret_cast<uint4 *>(row);
#pragma unroll
                    for (int e = 0; e < CPT / 8; ++e)
                        dst[e] = make_uint4(pack_bf16(o[8 * e], o[8 * e + 1]), pack_bf16(o[8 * e + 2], o[8 * e + 3]),
                                            pack_bf16(o[8 * e + 4], o[8 * e + 5]), pack_bf16(o[8 * e + 6], o[8 * e + 7]));
                }
            }
            return true;
        };
        write_B1(0);
        tc_fence_before();
        bool failed = false, ok = true;
        for (int i = 0; i < nchunks; ++i) {
            const int s = i % NS;
            const int p = i & 1;
            const unsigned char *st = sm + (size_t)s * L::STAGE;
            if (named_bar_or(BAR_S, NSYNC, !ok)) { failed = true; break; }
            // this chunk's stage has landed (the issuer saw it before the barrier);
            // U and e^{G_C} are read straight from it
            ok = mbar_wait(&full[s], (i / NS) & 1);
            const float eg = reinterpret_cast<const float *>(st + L::EGC_OFF)[t];
            uint32_t u[CPT / 2];
            if (t < 64) {
                // column (n0 % 32) + cb + c of the loaded U tile(s), row t
#pragma unroll
                for (int c = 0; c < CPT; c += 8) {
                    const int lc = (n0 & 31) + cb + c;
                    const uint4 x = *reinterpret_cast<const uint4 *>(st + L::U_OFF + (lc >> 5) * 4096 + t * 64 + (lc & 31) * 2);
                    u[c / 2] = x.x; u[c / 2 + 1] = x.y; u[c / 2 + 2] = x.z; u[c / 2 + 3] = x.w;
                }
            }
            if (t >= 64) {
                // the previous chunk's output leaves through the lane 64-127
                // warps while MMA1 runs and the others form V_new (off the
                // sequential path)
                if (i > 0 && !emit_output(i - 1)) ok = false;
            } else {
                if (ok) ok = mbar_wait(mma1, i & 1);
                tc_fence_after();
                // V_new = U - W S for token row t
                float x[CPT];
                tmem_row(p * DVT, x);
#pragma unroll
                for (int ng = 0; ng < CPT / 8; ++ng) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 u2 = *reinterpret_cast<const __nv_bfloat162 *>(&u[4 * ng + e]);
                        pk[e] = pack_bf16(__low2float(u2) - x[8 * ng + 2 * e], __high2float(u2) - x[8 * ng + 2 * e + 1]);
                    }
                    *reinterpret_cast<uint4 *>(B2 + p * L::B2_BYTES + L::template b_off<L::B2_ATOM>(t, cb / 8 + ng)) =
                        make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    if (v_img) {
                        // the backward's V_new image [C][dv], K-major SW128
                        const int n = n0 + cb + 8 * ng;
                        *reinterpret_cast<uint4 *>(v_img + ((size_t)(max(c_begin, 0) + i) * H + h) * 16384 +
                                                   (size_t)(n >> 6) * 8192 + ws::sw128(t, n & 63)) =
                            make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            if (named_bar_or(BAR_V, NSYNC, !ok)) { failed = true; break; }
            ok = mbar_wait(mma3, i & 1);
            tc_fence_after();
            // S <- Diag(e^{G_C}) S + Kt^T V_new   (channel row t)
            {
                float z[CPT];
                tmem_row(2 * DVT, z);
#pragma unroll
                for (int e = 0; e < CPT; ++e) S[e] = eg * S[e] + z[e];
            }
            write_B1(i + 1);
            tc_fence_before();
        }
        if (!failed && !ok) failed = true;
        if (!failed && nchunks > 0 && t >= 64 && !emit_output(nchunks - 1)) failed = true;
        if (failed) {
            set_device_error(err, kErrWaitTimeout);
            *abort_flag = 1;
        } else if (sT) {
            const size_t sb = (((size_t)seq * H + h) * D + t) * D + n0 + cb;
#pragma unroll
            for (int j = 0; j < CPT; j += 4)
                *reinterpret_cast<float4 *>(sT + sb + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, L::NCOLS);
}

template <int DVT, int NS>
cudaError_t launch_tc(const unsigned char *wsp, const int32_t *cu, const int32_t *coff,
                      const float *s0, float *sT, void *out, int N, int T, int total_T, int H,
                      int max_chunks, int *err, cudaStream_t st, unsigned char *s_img,
                      unsigned char *v_img, const int32_t *order)
{
    using L = TcLayout<DVT, NS>;
    const size_t smem = L::BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(chunk_chain_tc_kernel<DVT, NS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(D / DVT, H, N);
    chunk_chain_tc_kernel<DVT, NS><<<grid, L::NTHREADS, smem, st>>>(
        wsp, cu, coff, s0, sT, (__nv_bfloat16 *)out, T, total_T, H, (T + C - 1) / C, max_chunks, err,
        s_img, v_img, order, ((uintptr_t)out & 31u) == 0);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_chain(const unsigned char *wsp, const int32_t *cu, const int32_t *coff,
                                  const float *s0, float *sT, void *out, int N, int T,
                                  int total_T, int H, int dvt, int max_chunks, int *err,
                                  cudaStream_t st, unsigned char *s_img, unsigned char *v_img,
                                  const int32_t *order)
{
#define KDA_CHAIN_ARGS wsp, cu, coff, s0, sT, out, N, T, total_T, H, max_chunks, err, st, s_img, v_img, order
    switch (dvt) {
        case 16: return launch_tc<16, 3>(KDA_CHAIN_ARGS);
        case 32: return launch_tc<32, 3>(KDA_CHAIN_ARGS);
        case 64: return launch_tc<64, 2>(KDA_CHAIN_ARGS);
        case 128: return launch_tc<128, 2>(KDA_CHAIN_ARGS);
    }
#undef KDA_CHAIN_ARGS
    return cudaErrorInvalidValue;
}

}  // namespace kda
