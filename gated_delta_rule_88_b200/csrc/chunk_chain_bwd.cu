// chunk_chain_bwd.cu -- reverse chain of the chunked KDA backward (bf16,
// dk = dv = 128, C = 64) on tcgen05.
//
// Reverse mode through the chunk form: with dS' the gradient of the state
// leaving chunk c (dS' = dS_T for the last chunk), per chunk from last to first
// and one DVT-column tile of the state gradient (dk x DVT, fp32 registers):
//     R0 (off the sequential path)  D1b = P^T dO           (M = 64, TMEM lanes +16)
//     R1                             D1a = Kt dS'           (M = 64, TMEM lanes +0)
//           dV_new = D1a + D1b      (token row per thread pair, summed by shuffle)
//     R2                             D3 = Qg^T dO + W^T (-dV_new)   (M = 128 channels)
//           dS <- Diag(e^{G_C}) dS' + D3
// and at the end dS is the gradient of the initial state.  Every A operand is
// read from the forward record as an MN-major operand (the record's K-major
// tiles transposed in place); B operands: dS' (bf16, written by the threads),
// -dV_new (bf16, written by the threads) and the dO tile (TMA, 64-byte swizzle).
// For the per-chunk pass the kernel stores, per (chunk, head), dS' and dV_new
// as bf16 K-major SW128 images ([dk][dv], [C][dv]; 64-column blocks).
//
// Roles (192 threads): warps 0-3 epilogue (thread t <-> TMEM lane t), warp 4
// lane 0 the loader (bulk copies of the record head and e^{G_C}, a TMA box of
// dO), warp 5 lane 0 the MMA issuer (its warp joins the named barriers).
#include "chunk_ws.h"
#include "common.cuh"
#include "kernels.h"
#include "prep_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;
constexpr int C = ws::C;
constexpr int D = ws::D;
constexpr uint32_t REC_HEAD = 57344;          // [W;Qg] + Kt^T + P

// image offsets (bytes) inside a (chunk, head) slot of the backward workspace
constexpr size_t DSP_BYTES = 32768;           // dS' [dk][dv] bf16, SW128 K-major, 2 blocks
constexpr size_t DVN_BYTES = 16384;           // dV_new [C][dv] bf16, SW128 K-major, 2 blocks

__host__ __device__ constexpr uint32_t idesc_bf16_mn(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct BwdLayout {
    static constexpr int DVT = 32;
    static constexpr int NS = 3;
    static constexpr uint32_t EGC_OFF = REC_HEAD;
    static constexpr uint32_t DO_OFF = 58368;                 // 1024-aligned, 64 x 64 B
    static constexpr uint32_t STAGE = DO_OFF + 4096;          // 62464
    static constexpr uint32_t TX = REC_HEAD + 512 + 4096;
    static constexpr uint32_t B1_OFF = NS * STAGE;            // dS' bf16: K = 128 x N = 32
    static constexpr uint32_t B2_OFF = B1_OFF + 128 * DVT * 2;   // -dV_new: K = 64 x N = 32
    static constexpr uint32_t BAR_OFF = B2_OFF + 64 * DVT * 2;
    static constexpr uint32_t BYTES = BAR_OFF + 8 * 16 + 16;
    static constexpr uint32_t NCOLS = 64;                     // D1 (32 cols, both lane halves) + D3
    static constexpr uint32_t BW = DVT * 2;                   // 64-byte rows, 64-byte swizzle
    static constexpr uint32_t B_SBO = 8 * BW;
    static constexpr uint32_t B_LAYOUT = 4;
    static __device__ __forceinline__ uint32_t b_off(int k, int chunk) {
        return (k >> 3) * B_SBO + (k & 7) * BW + ((chunk ^ ((((k & 7) * BW) >> 7) & 3)) << 4);
    }
};

__global__ void __launch_bounds__(192, 1)
chunk_chain_bwd_kernel(const __grid_constant__ CUtensorMap tm_do, const unsigned char *__restrict__ wsp,
                       const int32_t *__restrict__ cu, const int32_t *__restrict__ coff,
                       const float *__restrict__ dsT, float *__restrict__ ds0,
                       unsigned char *__restrict__ dsp_img, unsigned char *__restrict__ dvn_img,
                       int T, int total_T, int H, int cps, int max_chunks, int *__restrict__ err)
{
    using L = BwdLayout;
    constexpr int DVT = L::DVT, NS = L::NS;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::BAR_OFF);
    uint64_t *empty = full + NS;
    uint64_t *mma1 = empty + NS;       // R1 done
    uint64_t *mma2 = mma1 + 1;         // R0 done
    uint64_t *mma3 = mma1 + 2;         // R2 done
    uint64_t *drain = mma1 + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::BAR_OFF + 8 * 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    unsigned char *B1 = sm + L::B1_OFF;
    unsigned char *B2 = sm + L::B2_OFF;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n0 = blockIdx.x * DVT, h = blockIdx.y, seq = blockIdx.z;

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
    const int cb0 = max(c_begin, 0);
    // the r-th step handles chunk nchunks - 1 - r of the sequence
    auto rec_of = [&](int r) {
        return wsp + ((size_t)(cb0 + nchunks - 1 - r) * H + h) * ws::RECORD;
    };
    auto slot_of = [&](int r) { return (size_t)(cb0 + nchunks - 1 - r) * H + h; };

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        mbar_init(mma1, 1);
        mbar_init(mma2, 1);
        mbar_init(mma3, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(tmem_slot, L::NCOLS); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr int BAR_S = 1, BAR_V = 2;
    constexpr int NSYNC = 32 * 4 + 32;
    const uint32_t D1 = tmem, D3 = tmem + DVT;

    if (warp == 4) {
        // ---------------- loader ----------------
        if (lane == 0) {
            int issued = 0;
            for (int r = 0; r < nchunks; ++r) {
                const int s = r % NS;
                if (r >= NS && !mbar_wait(&empty[s], ((r / NS) - 1) & 1)) {
                    set_device_error(err, kErrWaitTimeout);
                    break;
                }
                if (*abort_flag) break;
                const unsigned char *rec = rec_of(r);
                unsigned char *st = sm + (size_t)s * L::STAGE;
                const long long tok0 = bos + (long long)C * (nchunks - 1 - r);
                mbar_arrive_expect_tx(&full[s], L::TX);
                bulk_g2s(st, rec, REC_HEAD, &full[s]);
                bulk_g2s(st + L::EGC_OFF, rec + ws::OFF_EGC, 512, &full[s]);
                prep::tma_load_3d(st + L::DO_OFF, &tm_do, n0, h, (int)tok0, &full[s]);
                issued = r + 1;
            }
            for (int j = max(0, issued - NS); j < issued; ++j)
                mbar_wait(&full[j % NS], (j / NS) & 1, 1u << 20);
        }
    } else if (warp == 5) {
        // ---------------- MMA issuer ----------------
        constexpr uint32_t ID64 = idesc_bf16_mn(64, DVT);
        constexpr uint32_t ID128 = idesc_bf16_mn(128, DVT);
        const uint32_t sa = smem_u32(sm);
        // MN-major SW128 A operands from the record: 64-element atoms along M,
        // 8-row K groups 1024 B apart (SBO), next 64-element atom (LBO)
        const DescParts a_kt = smem_desc_parts(sa + ws::OFF_KTT, 16384, 1024, 2);   // Kt: M = 64 tokens
        const DescParts a_pt = smem_desc_parts(sa + ws::OFF_P, 16384, 1024, 2);     // P^T: M = 64 tokens
        const DescParts a_qg = smem_desc_parts(sa + ws::OFF_AW + 8192, 16384, 1024, 2);  // Qg^T: M = 128 ch
        const DescParts a_w = smem_desc_parts(sa + ws::OFF_AW, 16384, 1024, 2);     // W^T: M = 128 ch
        const DescParts b_ds = smem_desc_parts(smem_u32(B1), L::B_SBO, L::B_SBO, L::B_LAYOUT);
        const DescParts b_dv = smem_desc_parts(smem_u32(B2), L::B_SBO, L::B_SBO, L::B_LAYOUT);
        const DescParts b_do = smem_desc_parts(sa + L::DO_OFF, L::B_SBO, L::B_SBO, L::B_LAYOUT);
        constexpr uint32_t BK = (2 * L::B_SBO) >> 4;   // B step per 16 K rows
        constexpr uint32_t AK = 2048 >> 4;              // A step per 16 K rows (two 8-row groups)
        bool issued_any = false;
        auto issue_r0 = [&](int r) -> bool {
            const int s = r % NS;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&full[s], (r / NS) & 1);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t so = ((uint32_t)s * L::STAGE) >> 4;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16_p(D1 + (16u << 16), a_pt.lo + so + kk * AK, a_pt.hi, b_do.lo + so + kk * BK,
                                b_do.hi, ID64, kk > 0);
                umma_commit(mma2);
            }
            __syncwarp();
            return true;
        };
        bool ok = nchunks > 0 ? issue_r0(0) : true;
        if (nchunks > 0) issued_any = true;
        for (int r = 0; r < nchunks; ++r) {
            const int s = r % NS;
            const uint32_t so = ((uint32_t)s * L::STAGE) >> 4;
            if (named_bar_or(BAR_S, NSYNC, !ok)) break;        // dS' is in B1
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16_p(D1, a_kt.lo + so + kk * AK, a_kt.hi, b_ds.lo + kk * BK, b_ds.hi, ID64, kk > 0);
                umma_commit(mma1);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16_p(D3, a_qg.lo + so + kk * AK, a_qg.hi, b_do.lo + so + kk * BK, b_do.hi, ID128,
                                kk > 0);
            }
            __syncwarp();
            if (named_bar_or(BAR_V, NSYNC, false)) break;      // -dV_new is in B2; D1 read
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16_p(D3, a_w.lo + so + kk * AK, a_w.hi, b_dv.lo + kk * BK, b_dv.hi, ID128, 1);
                umma_commit(mma3);
                umma_commit(&empty[s]);
            }
            __syncwarp();
            if (r + 1 < nchunks) ok = issue_r0(r + 1);
        }
        if (lane == 0 && issued_any) {
            umma_commit(drain);
            mbar_wait(drain, 0, 1u << 20);
        }
    } else {
        // ---------------- epilogue warps 0-3 ----------------
        const int t = tid;                                  // channel row of D3
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        // D1 rows: lanes 0-15 of warp w -> token 16w + lane (Kt dS'), lanes
        // 16-31 -> token 16w + lane - 16 (P^T dO)
        const int tok_row = 16 * warp + (lane & 15);
        const int half = lane >> 4;                         // which 16 columns this thread writes
        float dS[DVT];
        {
            const size_t sb = (((size_t)seq * H + h) * D + t) * D + n0;
#pragma unroll
            for (int j = 0; j < DVT; j += 4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (dsT) x = *reinterpret_cast<const float4 *>(dsT + sb + j);
                dS[j] = x.x; dS[j + 1] = x.y; dS[j + 2] = x.z; dS[j + 3] = x.w;
            }
        }
        // dS' -> B1 (bf16 operand) and the chunk's dS' image
        auto write_dsp = [&](int r) {
            unsigned char *img = dsp_img + slot_of(r) * DSP_BYTES;
#pragma unroll
            for (int ng = 0; ng < DVT / 8; ++ng) {
                const uint4 pk = make_uint4(pack_bf16(dS[8 * ng], dS[8 * ng + 1]), pack_bf16(dS[8 * ng + 2], dS[8 * ng + 3]),
                                            pack_bf16(dS[8 * ng + 4], dS[8 * ng + 5]), pack_bf16(dS[8 * ng + 6], dS[8 * ng + 7]));
                *reinterpret_cast<uint4 *>(B1 + L::b_off(t, ng)) = pk;
                const int n = n0 + 8 * ng;
                *reinterpret_cast<uint4 *>(img + (size_t)(n >> 6) * 16384 + ws::sw128(t, n & 63)) = pk;
            }
            fence_proxy_async_smem();
        };
        bool failed = false, ok = true;
        if (nchunks > 0) write_dsp(0);
        tc_fence_before();
        for (int r = 0; r < nchunks; ++r) {
            const int s = r % NS;
            const unsigned char *st = sm + (size_t)s * L::STAGE;
            if (named_bar_or(BAR_S, NSYNC, !ok)) { failed = true; break; }
            ok = mbar_wait(&full[s], (r / NS) & 1);
            const float eg = reinterpret_cast<const float *>(st + L::EGC_OFF)[t];
            if (ok) ok = mbar_wait(mma2, r & 1);
            if (ok) ok = mbar_wait(mma1, r & 1);
            tc_fence_after();
            {
                float x[DVT];
                tmem_ld32(D1 + lane_base, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < DVT; ++j) x[j] += __shfl_xor_sync(0xffffffffu, x[j], 16);
                // dV_new row tok_row, columns 16 half .. 16 half + 15
                unsigned char *img = dvn_img + slot_of(r) * DVN_BYTES;
                float y[16];                                    // this thread's 16 columns
#pragma unroll
                for (int j = 0; j < 16; ++j) y[j] = half ? x[16 + j] : x[j];
#pragma unroll
                for (int ng = 0; ng < 2; ++ng) {
                    const int c8 = 2 * half + ng;               // 8-column group in the tile
                    const float *xs = y + 8 * ng;
                    const uint4 neg = make_uint4(pack_bf16(-xs[0], -xs[1]), pack_bf16(-xs[2], -xs[3]),
                                                 pack_bf16(-xs[4], -xs[5]), pack_bf16(-xs[6], -xs[7]));
                    const uint4 pos = make_uint4(pack_bf16(xs[0], xs[1]), pack_bf16(xs[2], xs[3]),
                                                 pack_bf16(xs[4], xs[5]), pack_bf16(xs[6], xs[7]));
                    *reinterpret_cast<uint4 *>(B2 + L::b_off(tok_row, c8)) = neg;
                    const int n = n0 + 8 * c8;
                    *reinterpret_cast<uint4 *>(img + (size_t)(n >> 6) * 8192 + ws::sw128(tok_row, n & 63)) = pos;
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            if (named_bar_or(BAR_V, NSYNC, !ok)) { failed = true; break; }
            ok = mbar_wait(mma3, r & 1);
            tc_fence_after();
            {
                float z[DVT];
                tmem_ld32(D3 + lane_base, z);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < DVT; ++e) dS[e] = eg * dS[e] + z[e];
            }
            if (r + 1 < nchunks) write_dsp(r + 1);
            tc_fence_before();
        }
        if (!failed && !ok) failed = true;
        if (failed) {
            set_device_error(err, kErrWaitTimeout);
            *abort_flag = 1;
        } else if (ds0) {
            const size_t sb = (((size_t)seq * H + h) * D + t) * D + n0;
#pragma unroll
            for (int j = 0; j < DVT; j += 4)
                *reinterpret_cast<float4 *>(ds0 + sb + j) = make_float4(dS[j], dS[j + 1], dS[j + 2], dS[j + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, L::NCOLS);
}

}  // namespace

// dO tensor map: [total_T, H, 128] bf16, boxes {32 channels, 1 head, 64 tokens},
// 64-byte swizzle (the B-operand layout of a 32-column tile)
cudaError_t launch_chunk_chain_bwd(const void *dout, const unsigned char *wsp, const int32_t *cu,
                                   const int32_t *coff, const float *dsT, float *ds0,
                                   unsigned char *dsp_img, unsigned char *dvn_img, int N, int T,
                                   int total_T, int H, int max_chunks, int *err, cudaStream_t st)
{
    using L = BwdLayout;
    PFN_cuTensorMapEncodeTiled_v12000 enc = prep::tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap m;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)total_T};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)D * 2 * H};
    const cuuint32_t box[3] = {(cuuint32_t)L::DVT, 1, (cuuint32_t)C};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(dout), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const size_t smem = L::BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(chunk_chain_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(D / L::DVT, H, N);
    chunk_chain_bwd_kernel<<<grid, 192, smem, st>>>(m, wsp, cu, coff, dsT, ds0, dsp_img, dvn_img, T,
                                                     total_T, H, (T + C - 1) / C, max_chunks, err);
    return cudaGetLastError();
}

}  // namespace kda
