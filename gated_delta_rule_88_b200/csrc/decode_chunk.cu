// decode_chunk.cu -- the L-token KDA decode on a slot-indexed state pool in
// the chunk form, on tensor cores (bf16 operands, fp32 accumulation and
// state), dk = dv = 128.
//
// Kimi Linear paper notes (paper-notes-site): section 2 gives the recurrence,
// section 3 the chunkwise form (a WY-like representation of a chunk's
// writes, then one product with the fixed-size state).  For a block of up
// to 16 tokens of one (sequence, head), with G the block-local inclusive
// cumsum of g:
//     A_ij = beta_i sum_c k_ic k_jc e^{G_ic - G_jc}  (j < i)
//     P_ij =        sum_c q_ic k_jc e^{G_ic - G_jc}  (j <= i)
//     T = (I + A)^-1,  W = T (beta K e^G),  U = T (beta V)
//     V_new = U - W S;  O = (Q e^G) S + P V_new
//     S <- Diag(e^{G_last}) S + (K e^{G_last - G})^T V_new
// The same algebra as the chunked prefill.  A and P: when every g of the
// block is >= -5 (|G| <= 80 over 16 tokens) they are products of the forms
// beta k e^G, q e^G and k e^{-G} on tensor cores, as in the prefill; else
// they are formed directly from e^{G_i - G_j} <= 1 in fp32 (exact
// exponentials, no factorisation), so any finite g <= 0 is accepted.
//
// Persistent CTAs (256 threads, 8 warps, one per SM) walk the (sequence,
// head) items.  The fp32 state lives in registers in the m16n8k16
// accumulator layout (warp w: channel rows 16w .. 16w + 15, all 128
// columns), so the state update is one tensor-core accumulate into it; its
// bf16 copy in shared memory is the B operand of W S and (Q e^G) S.  While an
// item runs, each thread's share of the next item's state arrives by
// cp.async in a thread-private shared-memory slot, and the next block's token
// rows likewise.  Rounding: the MMA operands (S, V_new, T, P and the decayed
// forms) are bf16, as in the prefill.
#include "common.cuh"
#include "kernels.h"
#include "prep_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

constexpr int NT = 256;
constexpr int D = 128;
constexpr int BT = 16;                       // tokens per block (one MMA row tile)
constexpr float LOG2E = 1.4426950408889634f;

// 16 or 128 rows x 128 bf16, 256-byte rows, 16-byte chunk j of row r at j ^ (r & 7)
__device__ __forceinline__ int toff(int r, int c) {
    return r * 256 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1);
}
__device__ __forceinline__ int toff_chunk(int r, int j) { return r * 256 + (((j ^ (r & 7))) << 4); }

// shared-memory layout (bytes)
constexpr int OFF_RQ = 0;                    // raw q [16][128] bf16, 256-byte rows
constexpr int OFF_RK = OFF_RQ + 4096;
constexpr int OFF_RV = OFF_RK + 4096;
constexpr int OFF_G = OFF_RV + 4096;         // g, then log2e * cumsum, fp32 [16][128]
constexpr int OFF_BETA = OFF_G + 8192;       // [16] fp32 (128 bytes reserved)
constexpr int OFF_QG = OFF_BETA + 128;       // forms: [16][128] bf16, toff layout
constexpr int OFF_KG = OFF_QG + 4096;        // beta k e^G
constexpr int OFF_KT = OFF_KG + 4096;        // k e^{G_last - G}
constexpr int OFF_BV = OFF_KT + 4096;        // beta v
constexpr int OFF_W = OFF_BV + 4096;         // W = T (beta k e^G)
constexpr int OFF_VN = OFF_W + 4096;         // V_new
constexpr int OFF_SB = OFF_VN + 4096;        // state copy [128][128] bf16, toff layout
constexpr int OFF_AM = OFF_SB + 32768;       // A, P, T: fp32 [16][16]
constexpr int OFF_PM = OFF_AM + 1024;
constexpr int OFF_TM = OFF_PM + 1024;
constexpr int OFF_GAM = OFF_TM + 1024;       // e^{G_last} per channel, fp32 [128]
constexpr int OFF_KD = OFF_GAM + 512;        // k e^{-G} (factorised A and P)
constexpr int OFF_SN = OFF_KD + 4096;        // next item's state, fp32 [128][128], fsw layout
constexpr int OFF_SO = OFF_SN + D * D * 4;   // finished item's state on its way out, fsw layout
constexpr int OFF_BAR = OFF_SO + D * D * 4;  // mbarrier of the raw rows
constexpr int SMEM = OFF_BAR + 16;
constexpr uint32_t TX_RAW = 3 * 4096 + 8192;   // q, k, v, g rows of one block
static_assert(OFF_QG % 16 == 0 && OFF_SB % 16 == 0 && OFF_KD % 16 == 0 && OFF_SN % 16 == 0 &&
              OFF_BAR % 8 == 0 && SMEM <= 227 * 1024, "layout");

// 2^x by the hardware approximation (PTX ex2.approx.ftz: relative error about
// 2^-22, results below 2^-126 flush to zero); the operands of the products it
// feeds are rounded to bf16 (2^-9).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void cp_async4_zfill(void *smem_dst, const void *gmem_src, bool ok) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(smem_u32(smem_dst)),
                 "l"(gmem_src), "r"(ok ? 4 : 0));
}
// fp32 [128][128] state in shared memory: 16-byte chunk j of row r at
// j ^ 2 (r & 3), so that a half-warp reading accumulator pairs (rows
// 16w + gid, gid = 0..3) and a warp copying one whole row are conflict-free
__device__ __forceinline__ int fsw(int r, int c) {
    return r * 512 + ((((c >> 2) ^ (2 * (r & 3)))) << 4) + ((c & 3) << 2);
}

// A fragment (rows gid / gid + 8, k pairs) of a 16 x 16 fp32 matrix in shared memory
__device__ __forceinline__ void frag16(uint32_t (&a)[4], const float *M, int gid, int tig) {
    const float2 x0 = *reinterpret_cast<const float2 *>(M + gid * 16 + 2 * tig);
    const float2 x1 = *reinterpret_cast<const float2 *>(M + (gid + 8) * 16 + 2 * tig);
    const float2 x2 = *reinterpret_cast<const float2 *>(M + gid * 16 + 2 * tig + 8);
    const float2 x3 = *reinterpret_cast<const float2 *>(M + (gid + 8) * 16 + 2 * tig + 8);
    a[0] = pack_bf16(x0.x, x0.y);
    a[1] = pack_bf16(x1.x, x1.y);
    a[2] = pack_bf16(x2.x, x2.y);
    a[3] = pack_bf16(x3.x, x3.y);
}

// Tensor map over a [rows, H, 128] token tensor of `elem`-byte elements,
// boxes of one head's 16 token rows (no swizzle: plain 128-element rows)
cudaError_t make_block_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem, int H,
                           int rows) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = prep::tensor_map_encoder();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)D * elem, (cuuint64_t)D * elem * H};
    const cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)BT};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

__global__ void __launch_bounds__(NT, 1)
decode_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                    const float *__restrict__ beta, float *__restrict__ pool,
                    const int32_t *__restrict__ slots, int num_slots,
                    __nv_bfloat16 *__restrict__ out, int N, int H, int L,
                    const int2 *__restrict__ list, const int *__restrict__ list_count, int *__restrict__ err)
{
    extern __shared__ __align__(128) unsigned char sm[];
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const int items = N * H;
    float *Gs = reinterpret_cast<float *>(sm + OFF_G);
    float *bs = reinterpret_cast<float *>(sm + OFF_BETA);
    float *Am = reinterpret_cast<float *>(sm + OFF_AM);
    float *Pm = reinterpret_cast<float *>(sm + OFF_PM);
    float *Tm = reinterpret_cast<float *>(sm + OFF_TM);
    float *gam = reinterpret_cast<float *>(sm + OFF_GAM);
    const int nblk = (L + BT - 1) / BT;
    // the next item at or after `it` (grid stride) with a valid slot; -1 if
    // none.  Every thread walks the same items, so the answer is uniform.
    // With a list, the walk is over list entries (item, first token, a
    // multiple of 64) instead of items; listed items have valid slots.
    const int n_list = list ? *list_count : 0;
    auto item_of = [&](int ix) -> int { return list ? list[ix].x : ix; };
    auto first_blk = [&](int ix) -> int { return list ? list[ix].y / BT : 0; };
    auto next_valid = [&](int it) -> int {
        if (list) return it < n_list ? it : -1;
        for (; it < items; it += gridDim.x) {
            const int nn = it / H;
            const int sl = slots ? slots[nn] : nn;
            if (sl >= 0 && sl < num_slots) return it;
            if (tid == 0) set_device_error(err, kErrBadSlot);
        }
        return -1;
    };
    auto state_of = [&](int it) -> float * {
        const int nn = it / H, hh = it - nn * H;
        const int sl = slots ? slots[nn] : nn;
        return pool + ((size_t)sl * H + hh) * (size_t)(D * D);
    };
    // token l of item `it` is row row0(it) + l * H of the token arrays
    auto row0 = [&](int it) -> size_t {
        const int nn = it / H, hh = it - nn * H;
        return (size_t)nn * L * H + hh;
    };

    // raw rows of block b of item `it`: q, k, v and g by TMA (16 token rows
    // of one head; rows past the item's last token hold whatever follows and
    // are masked where they are read), beta by cp.async (zero past the last
    // token), one cp.async group
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    auto issue_raw = [&](int it, int b) {
        const int l0 = b * BT, nt = min(BT, L - l0);
        const int nn = it / H, hh = it - nn * H;
        if (tid == 0) {
            const int row = nn * L + l0;
            sm100::mbar_arrive_expect_tx(bar, TX_RAW);
            prep::tma_load_3d(sm + OFF_RQ, &tm_q, 0, hh, row, bar);
            prep::tma_load_3d(sm + OFF_RK, &tm_k, 0, hh, row, bar);
            prep::tma_load_3d(sm + OFF_RV, &tm_v, 0, hh, row, bar);
            prep::tma_load_3d(sm + OFF_G, &tm_g, 0, hh, row, bar);
        }
        const size_t base = row0(it);
        if (tid < BT) cp_async4_zfill(bs + tid, beta + base + (size_t)(tid < nt ? l0 + tid : l0) * H, tid < nt);
        cp_async_commit();
    };
    uint32_t raw_phase = 0;    // parity of the raw-row barrier's next completion

    // the state, fp32, in the accumulator layout: s[j] = rows (16w + gid,
    // 16w + gid + 8) x columns (8j + 2tig, + 1).  Element pair (j, half) of
    // thread t has its own 8-byte slot in the prefetch area.
    const int r0 = 16 * w + gid, r1 = r0 + 8;
    // the next item's state: whole rows (one per warp and instruction) into
    // the fsw layout; joins the next committed group
    auto issue_state = [&](int it) {
        const float *Sg = state_of(it);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int idx = e * NT + tid, r = idx >> 5, c = 4 * (idx & 31);
            cp_async16(sm + OFF_SN + fsw(r, c), Sg + (size_t)r * D + c);
        }
    };
    float s[16][4];
    auto write_sb = [&]() {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            *reinterpret_cast<uint32_t *>(sm + OFF_SB + toff(r0, 8 * j + 2 * tig)) = pack_bf16(s[j][0], s[j][1]);
            *reinterpret_cast<uint32_t *>(sm + OFF_SB + toff(r1, 8 * j + 2 * tig)) = pack_bf16(s[j][2], s[j][3]);
        }
    };

    if (tid == 0) {
        sm100::mbar_init(bar, 1);
        sm100::fence_mbar_init();
    }
    __syncthreads();
    int cur = next_valid(blockIdx.x);
    if (cur < 0) return;
    issue_state(item_of(cur));
    issue_raw(item_of(cur), first_blk(cur));
    while (cur >= 0) {
    const int nxt = next_valid(cur + gridDim.x);
    const int cit = item_of(cur), b_first = first_blk(cur);
    const size_t orow = row0(cit);
    for (int b = b_first; b < nblk; ++b) {
        const int l0 = b * BT, nt = min(BT, L - l0);
        cp_async_wait<0>();
        bool ok = true;
        if (tid == 0) ok = sm100::mbar_wait(bar, raw_phase);
        raw_phase ^= 1u;
        if (!__syncthreads_and(ok)) {
            // the raw rows never arrived: report, give the copy a bounded
            // second wait, and stop before shared memory is released
            if (tid == 0) {
                set_device_error(err, kErrWaitTimeout);
                sm100::mbar_wait(bar, raw_phase ^ 1u);
            }
            return;
        }                                      // raw rows of block b (and at b = 0 the state) landed
        if (b == b_first) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float2 x = *reinterpret_cast<const float2 *>(sm + OFF_SN + fsw(r0, 8 * j + 2 * tig));
                const float2 y = *reinterpret_cast<const float2 *>(sm + OFF_SN + fsw(r1, 8 * j + 2 * tig));
                s[j][0] = x.x; s[j][1] = x.y; s[j][2] = y.x; s[j][3] = y.y;
            }
            write_sb();
        }

        // 1. per channel: log2e-scaled inclusive cumsum of g (in place), the
        //    block decay; meanwhile the other threads clear A and P
        bool in_range = true;
        if (tid < D) {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < BT; ++i) {
                const float gv = i < nt ? Gs[i * D + tid] : 0.f;
                in_range = in_range && gv >= -5.f;
                acc = fmaf(gv, LOG2E, acc);
                Gs[i * D + tid] = acc;
            }
            gam[tid] = ex2(acc);
        } else {
            for (int e = tid - D; e < 512; e += NT - D) (e < 256 ? Am : Pm)[e & 255] = 0.f;
        }
        // factorised A and P when every g of the block is >= -5
        const bool fact = __syncthreads_and(in_range);

        // 2. decayed forms (thread: token i, channel pair), A and P
        for (int it = tid; it < BT * 64; it += NT) {
            const int i = it >> 6, c = 2 * (it & 63);
            const float2 gi = *reinterpret_cast<const float2 *>(Gs + i * D + c);
            const float2 gl = *reinterpret_cast<const float2 *>(Gs + (BT - 1) * D + c);
            const float ex = ex2(gi.x), ey = ex2(gi.y);
            const float tx = ex2(gl.x - gi.x), ty = ex2(gl.y - gi.y);
            const bool row_ok = i < nt;
            const __nv_bfloat162 zero2 = __floats2bfloat162_rn(0.f, 0.f);
            const __nv_bfloat162 q2 = row_ok ? *reinterpret_cast<const __nv_bfloat162 *>(sm + OFF_RQ + i * 256 + 2 * c) : zero2;
            const __nv_bfloat162 k2 = row_ok ? *reinterpret_cast<const __nv_bfloat162 *>(sm + OFF_RK + i * 256 + 2 * c) : zero2;
            const __nv_bfloat162 v2 = row_ok ? *reinterpret_cast<const __nv_bfloat162 *>(sm + OFF_RV + i * 256 + 2 * c) : zero2;
            const float b_ = bs[i];
            const float qx = __low2float(q2), qy = __high2float(q2);
            const float kx = __low2float(k2), ky = __high2float(k2);
            const int o = toff(i, c);
            *reinterpret_cast<uint32_t *>(sm + OFF_QG + o) = pack_bf16(qx * ex, qy * ey);
            *reinterpret_cast<uint32_t *>(sm + OFF_KG + o) = pack_bf16(b_ * kx * ex, b_ * ky * ey);
            *reinterpret_cast<uint32_t *>(sm + OFF_KT + o) = pack_bf16(kx * tx, ky * ty);
            *reinterpret_cast<uint32_t *>(sm + OFF_BV + o) =
                pack_bf16(b_ * __low2float(v2), b_ * __high2float(v2));
            if (fact) *reinterpret_cast<uint32_t *>(sm + OFF_KD + o) = pack_bf16(__fdividef(kx, ex), __fdividef(ky, ey));
        }
        if (!fact) {
            // pairs j <= i < nt, eight slices each; slice sl of pair p takes
            // channel pairs 2 sl + 16 m (m = 0..7), visited from a per-pair
            // rotation so that the four pairs of a warp read different banks.
            // The slices of a pair sit in eight consecutive lanes and meet by
            // shuffles.
            const int npairs = nt * (nt + 1) / 2;
            for (int base = 0; base < npairs * 8; base += NT) {
                const int it = base + tid;
                const bool valid = it < npairs * 8;
                const int p = valid ? it >> 3 : 0, sl = it & 7;
                int i = 0;
                while ((i + 1) * (i + 2) / 2 <= p) ++i;
                const int j = p - i * (i + 1) / 2;
                float a = 0.f, pp = 0.f;
                if (valid) {
                    const float *gi = Gs + i * D, *gj = Gs + j * D;
                    const unsigned char *qi = sm + OFF_RQ + i * 256, *ki = sm + OFF_RK + i * 256;
                    const unsigned char *kj = sm + OFF_RK + j * 256;
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const int c = 16 * ((m + p) & 7) + 2 * sl;
                        const float2 x = *reinterpret_cast<const float2 *>(gi + c);
                        const float2 y = *reinterpret_cast<const float2 *>(gj + c);
                        const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162 *>(qi + 2 * c);
                        const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162 *>(ki + 2 * c);
                        const __nv_bfloat162 l2 = *reinterpret_cast<const __nv_bfloat162 *>(kj + 2 * c);
                        const float e0 = ex2(x.x - y.x), e1 = ex2(x.y - y.y);
                        const float kj0 = __low2float(l2), kj1 = __high2float(l2);
                        a = fmaf(__low2float(k2) * kj0, e0, a);
                        a = fmaf(__high2float(k2) * kj1, e1, a);
                        pp = fmaf(__low2float(q2) * kj0, e0, pp);
                        pp = fmaf(__high2float(q2) * kj1, e1, pp);
                    }
                }
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) {
                    a += __shfl_xor_sync(0xffffffffu, a, o);
                    pp += __shfl_xor_sync(0xffffffffu, pp, o);
                }
                if (valid && sl == 0) {
                    if (j < i) Am[i * 16 + j] = bs[i] * a;
                    Pm[i * 16 + j] = pp;
                }
            }
        }
        // the in-place cumsum wrote g rows that the next TMA overwrites
        sm100::fence_proxy_async_smem();
        __syncthreads();
        if (fact) {
            // A = (beta k e^G)(k e^{-G})^T, P = (q e^G)(k e^{-G})^T: warps
            // 0-1 A, 2-3 P, one 8-column tile each
            if (w < 4) {
                const unsigned char *X = sm + (w < 2 ? OFF_KG : OFF_QG);
                const int nt8 = w & 1;
                const int ar = (lane & 7) + 8 * ((lane >> 3) & 1);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    uint32_t af[4], bf[2];
                    ldsm_x4(af, X + toff_chunk(ar, 2 * ks + (lane >> 4)));
                    // B (k = channel, n = token j) from k e^{-G} stored [token][channel]
                    bf[0] = *reinterpret_cast<const uint32_t *>(sm + OFF_KD + toff(8 * nt8 + gid, 16 * ks + 2 * tig));
                    bf[1] = *reinterpret_cast<const uint32_t *>(sm + OFF_KD + toff(8 * nt8 + gid, 16 * ks + 8 + 2 * tig));
                    mma_bf16(acc, af, bf[0], bf[1]);
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int i = gid + 8 * hh, j = 8 * nt8 + 2 * tig;
                    const float v0 = acc[2 * hh], v1 = acc[2 * hh + 1];
                    if (w < 2) {
                        Am[i * 16 + j] = (j < i) ? v0 : 0.f;
                        Am[i * 16 + j + 1] = (j + 1 < i) ? v1 : 0.f;
                    } else {
                        Pm[i * 16 + j] = (j <= i) ? v0 : 0.f;
                        Pm[i * 16 + j + 1] = (j + 1 <= i) ? v1 : 0.f;
                    }
                }
            }
            __syncthreads();
        }
        // the raw rows are dead: the next block's (or the next item's first
        // block's) arrive while this one runs
        if (b + 1 < nblk) issue_raw(cit, b + 1);
        else if (nxt >= 0) issue_raw(item_of(nxt), first_blk(nxt));

        // 3. T = (I + A)^-1 by forward substitution, one column per thread
        if (tid < BT) {
            // row i of A arrives as four vector loads before its two
            // interleaved accumulation chains (even and odd j)
            float x[BT];
#pragma unroll
            for (int i = 0; i < BT; ++i) {
                float ar[BT];
#pragma unroll
                for (int c4 = 0; c4 < BT / 4; ++c4) {
                    const float4 t4 = *reinterpret_cast<const float4 *>(Am + i * 16 + 4 * c4);
                    ar[4 * c4] = t4.x; ar[4 * c4 + 1] = t4.y; ar[4 * c4 + 2] = t4.z; ar[4 * c4 + 3] = t4.w;
                }
                float e0 = 0.f, e1 = 0.f;
#pragma unroll
                for (int j = 0; j < i; ++j) {
                    if (j & 1) e1 = fmaf(ar[j], x[j], e1);
                    else e0 = fmaf(ar[j], x[j], e0);
                }
                x[i] = (i < tid) ? 0.f : (i == tid) ? 1.f : -(e0 + e1);
            }
#pragma unroll
            for (int i = 0; i < BT; ++i) Tm[i * 16 + tid] = x[i];
        }
        __syncthreads();
        // every thread's reads of its state slots are long complete (several
        // barriers): the next item's state may now land there
        if (b == b_first && nxt >= 0) {
            issue_state(item_of(nxt));
            cp_async_commit();
        }

        // 4. W = T (beta k e^G) (channel tiles 2w, 2w + 1) and U = T (beta v)
        //    (value tiles 2w, 2w + 1; kept in registers)
        const int kr = (lane & 7) + 8 * ((lane >> 3) & 1);
        float u[2][4] = {}, wm[2][4] = {};
        {
            uint32_t ta[4], bf[4];
            frag16(ta, Tm, gid, tig);
            ldsm_x4_t(bf, sm + OFF_KG + toff_chunk(kr, 2 * w + (lane >> 4)));
            mma_bf16(wm[0], ta, bf[0], bf[1]);
            mma_bf16(wm[1], ta, bf[2], bf[3]);
            ldsm_x4_t(bf, sm + OFF_BV + toff_chunk(kr, 2 * w + (lane >> 4)));
            mma_bf16(u[0], ta, bf[0], bf[1]);
            mma_bf16(u[1], ta, bf[2], bf[3]);
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int c = 16 * w + 8 * jj + 2 * tig;
                *reinterpret_cast<uint32_t *>(sm + OFF_W + toff(gid, c)) = pack_bf16(wm[jj][0], wm[jj][1]);
                *reinterpret_cast<uint32_t *>(sm + OFF_W + toff(gid + 8, c)) = pack_bf16(wm[jj][2], wm[jj][3]);
            }
        }
        __syncthreads();

        // 5. W S and (q e^G) S for value tiles 2w, 2w + 1; V_new = U - W S
        float ws[2][4] = {}, os[2][4] = {};
        {
            const int ar = (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t aw[4], aq[4], bf[4];
                ldsm_x4_t(bf, sm + OFF_SB + toff_chunk(16 * ks + kr, 2 * w + (lane >> 4)));
                ldsm_x4(aw, sm + OFF_W + toff_chunk(ar, 2 * ks + (lane >> 4)));
                ldsm_x4(aq, sm + OFF_QG + toff_chunk(ar, 2 * ks + (lane >> 4)));
                mma_bf16(ws[0], aw, bf[0], bf[1]);
                mma_bf16(ws[1], aw, bf[2], bf[3]);
                mma_bf16(os[0], aq, bf[0], bf[1]);
                mma_bf16(os[1], aq, bf[2], bf[3]);
            }
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int c = 16 * w + 8 * jj + 2 * tig;
                *reinterpret_cast<uint32_t *>(sm + OFF_VN + toff(gid, c)) =
                    pack_bf16(u[jj][0] - ws[jj][0], u[jj][1] - ws[jj][1]);
                *reinterpret_cast<uint32_t *>(sm + OFF_VN + toff(gid + 8, c)) =
                    pack_bf16(u[jj][2] - ws[jj][2], u[jj][3] - ws[jj][3]);
            }
        }
        __syncthreads();

        // 6. O = (q e^G) S + P V_new for value tiles 2w, 2w + 1
        {
            uint32_t pa[4], bf[4];
            frag16(pa, Pm, gid, tig);
            ldsm_x4_t(bf, sm + OFF_VN + toff_chunk(kr, 2 * w + (lane >> 4)));
            mma_bf16(os[0], pa, bf[0], bf[1]);
            mma_bf16(os[1], pa, bf[2], bf[3]);
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int c = 16 * w + 8 * jj + 2 * tig;
                if (gid < nt)
                    *reinterpret_cast<uint32_t *>(out + (orow + (size_t)(l0 + gid) * H) * D + c) = pack_bf16(os[jj][0], os[jj][1]);
                if (gid + 8 < nt)
                    *reinterpret_cast<uint32_t *>(out + (orow + (size_t)(l0 + gid + 8) * H) * D + c) = pack_bf16(os[jj][2], os[jj][3]);
            }
        }

        // 7. S <- Diag(e^{G_last}) S + (k e^{G_last - G})^T V_new: channel rows
        //    16w .. 16w + 15, all value tiles, accumulated into the registers
        {
            const float g0 = gam[r0], g1 = gam[r1];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                s[j][0] *= g0; s[j][1] *= g0; s[j][2] *= g1; s[j][3] *= g1;
            }
            uint32_t ka[4];
            ldsm_x4_t(ka, sm + OFF_KT + toff_chunk((lane & 7) + 8 * (lane >> 4), 2 * w + ((lane >> 3) & 1)));
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bf[4];
                ldsm_x4_t(bf, sm + OFF_VN + toff_chunk(kr, 2 * np + (lane >> 4)));
                mma_bf16(s[2 * np], ka, bf[0], bf[1]);
                mma_bf16(s[2 * np + 1], ka, bf[2], bf[3]);
            }
        }
        // every warp has finished reading the old copy (step 5 precedes the
        // barrier after V_new); write the new one for the next block
        if (b + 1 < nblk) write_sb();
    }
    {
        // out through shared memory, so that each store instruction writes
        // whole rows
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            *reinterpret_cast<float2 *>(sm + OFF_SO + fsw(r0, 8 * j + 2 * tig)) = make_float2(s[j][0], s[j][1]);
            *reinterpret_cast<float2 *>(sm + OFF_SO + fsw(r1, 8 * j + 2 * tig)) = make_float2(s[j][2], s[j][3]);
        }
        __syncthreads();
        float *Sg = state_of(cit);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int idx = e * NT + tid, r = idx >> 5, c = 4 * (idx & 31);
            __stcs(reinterpret_cast<float4 *>(Sg + (size_t)r * D + c),
                   *reinterpret_cast<const float4 *>(sm + OFF_SO + fsw(r, c)));
        }
    }
    cur = nxt;
    }
}

namespace {
cudaError_t launch_walk(const void *q, const void *k, const void *v, const float *g, const float *beta,
                        float *pool, const int32_t *slots, int num_slots, void *out, int N, int H, int L,
                        const int2 *list, const int *list_count, int *err, cudaStream_t st)
{
    if (N == 0 || L == 0) return cudaSuccess;
    static int grid_for[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (grid_for[dev] == 0) {
        e = cudaFuncSetAttribute(decode_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
        if (e != cudaSuccess) return e;
        int sms = 0, per_sm = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_chunk_kernel, NT, SMEM)) != cudaSuccess)
            return e;
        grid_for[dev] = sms * (per_sm > 0 ? per_sm : 1);
    }
    const int items = N * H;
    const int grid = items < grid_for[dev] ? items : grid_for[dev];
    // [N * L token rows, H, 128] views, boxes of one head's 16 token rows
    if ((long long)N * L > 0x7fffffffLL) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mg;
    const int rows = N * L;
    e = make_block_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, rows);
    if (e == cudaSuccess) e = make_block_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, rows);
    if (e == cudaSuccess) e = make_block_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, rows);
    if (e == cudaSuccess) e = make_block_map(&mg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, rows);
    if (e != cudaSuccess) return e;
    decode_chunk_kernel<<<grid, NT, SMEM, st>>>(mq, mk, mv, mg, beta, pool, slots, num_slots,
                                                (__nv_bfloat16 *)out, N, H, L, list, list_count, err);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_decode_chunk(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float *pool, const int32_t *slots,
                                int num_slots, void *out, int N, int H, int L, int *err,
                                cudaStream_t st)
{
    return launch_walk(q, k, v, g, beta, pool, slots, num_slots, out, N, H, L, nullptr, nullptr, err, st);
}

cudaError_t launch_decode_chunk_list(const void *q, const void *k, const void *v, const float *g,
                                     const float *beta, float *pool, const int32_t *slots, int num_slots,
                                     void *out, int N, int H, int L, const int2 *list, const int *list_count,
                                     int *err, cudaStream_t st)
{
    return launch_walk(q, k, v, g, beta, pool, slots, num_slots, out, N, H, L, list, list_count, err, st);
}

}  // namespace kda
