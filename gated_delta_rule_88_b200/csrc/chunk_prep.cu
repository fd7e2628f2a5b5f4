// chunk_prep.cu -- per-(chunk, head) intra-chunk work of the bf16 KDA prefill
// (dk = dv = 128, C = 64).  Fully parallel over (chunk, head); no state.
//
// Kimi Linear paper notes (paper-notes-site), section 3: inside a chunk the
// intra-chunk writes are gathered by a WY-like representation (W, U) and the
// output splits into an inter-chunk and an intra-chunk part; section 2 and
// the constrained-DPLR remark: KDA ties the low-rank factors to k, which saves
// matrix products and avoids the inverse cumulative-decay (1/Gamma) terms of
// the general DPLR form.  This kernel produces, for one chunk of one head,
// the record of chunk_ws.h:
//     G     = chunk-local inclusive cumsum of g          (per channel)
//     A_ij  = beta_i sum_c k_ic k_jc e^{G_ic - G_jc}     (j < i)
//     P_ij  =        sum_c q_ic k_jc e^{G_ic - G_jc}     (j <= i)
//     T     = (I + A)^-1                                  (unit lower-tri.)
//     W = T (beta K e^G),  U = T (beta V),  Qg = Q e^G,  Kt = K e^{G_C - G}
//
// Exponents (no overflow, no 1/Gamma over the chunk): the chunk is cut into
// four sub-chunks of 16 tokens, I = 0..3, with block-end cumsums R_I
// (R_{-1} = 0).  For token i in block I and j in block J <= I,
//     e^{G_i - G_j} = e^{G_i - R_{I-1}} * e^{R_{I-1} - G_j}
// The left factor a_i = e^{G_i - R_{I-1}} is <= 1 and depends on i only;
// the right factor is <= 1 for J < I and spans at most 16 tokens for J = I,
// so with per-token g >= -5 every factor stays within e^{+-80}.  Row block I
// therefore needs one right operand Kr^(I)_j = k_j e^{R_{I-1} - G_j}
// (j < 16(I+1)); the four are stacked in shared memory.
//
// Tensor cores: m16n8k16 bf16 MMAs with fp32 accumulation for A, P (left
// operands (beta k a), (q a); right operand Kr^(I)), and W, U (T rounded to
// bf16 times (beta K e^G), (beta V)).  T itself is formed in fp32:
// 16x16 diagonal blocks by forward substitution, off-diagonal blocks by
// T_IJ = -T_II sum_{M=J}^{I-1} A_IM T_MJ in order of distance I - J.
#include "chunk_ws.h"
#include "common.cuh"
#include "kernels.h"

namespace kda {
namespace {

constexpr int C = ws::C;
constexpr int D = ws::D;
constexpr int NT = 256;
constexpr int PB = D + 8;     // bf16 pitch of 128-wide tiles (conflict-free ldmatrix)
constexpr int PF = C + 4;     // fp32 pitch of 64x64 tiles
constexpr int PP = C + 8;     // bf16 pitch of the 64x64 P staging tile
constexpr int KR_ROWS = 16 + 32 + 48 + 64;
__host__ __device__ constexpr int kr_base(int I) { return I == 0 ? 0 : I == 1 ? 16 : I == 2 ? 48 : 96; }

struct PrepSmem {
    union {
        float G[C][D];                        // cumsum of g (phase 1-3)
        __nv_bfloat16 Pst[C][PP];             // P staging (phase 4-7)
    };
    __nv_bfloat16 Xk[C][PB];                  // beta k a      (then W staging)
    __nv_bfloat16 Xq[C][PB];                  // q a           (then U staging)
    __nv_bfloat16 KG[C][PB];                  // beta k e^G
    __nv_bfloat16 Vb[C][PB];                  // beta v
    __nv_bfloat16 Kr[KR_ROWS][PB];            // k e^{R_{I-1} - G_j}, I = 0..3 stacked
    float A[C][PF];                           // A (strict lower), fp32
    float Tm[C][PF];                          // T, fp32
    float Zs[4][16][17];                      // per-warp 16x16 scratch
    float R[4][D];                            // block-end cumsums
    float Eb[4][D];                           // e^{R_{I-1}} (Eb[0] = 1)
    float F[4][D];                            // e^{R_3 - R_I}
    float Dm[16][D];                          // e^{R_{I'-1} - R_I}, index I*4+I', I < I'
    float beta[C];
};

__device__ __forceinline__ void locate_chunk(int chunk, const int32_t *cu, const int32_t *coff,
                                             int N, int T, int total_T, int cps, int &seq,
                                             long long &t0, int &len) {
    long long bos, eos;
    int cidx;
    if (cu) {
        int lo = 0, hi = N;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (coff[mid] <= chunk) lo = mid; else hi = mid;
        }
        seq = lo;
        bos = min(max(cu[seq], 0), total_T);
        eos = min(max(cu[seq + 1], 0), total_T);
        if (eos < bos) eos = bos;
        cidx = chunk - coff[seq];
    } else {
        seq = chunk / cps;
        cidx = chunk - seq * cps;
        bos = (long long)seq * T;
        eos = bos + T;
    }
    t0 = bos + (long long)C * cidx;
    len = (int)max(0LL, min((long long)C, eos - t0));
}

__global__ void __launch_bounds__(NT, 1)
chunk_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                  const __nv_bfloat16 *__restrict__ v, const float *__restrict__ g,
                  const float *__restrict__ beta, const int32_t *__restrict__ cu,
                  const int32_t *__restrict__ coff, int N, int T, int total_T, int H, int cps,
                  unsigned char *__restrict__ wsp)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    PrepSmem &sm = *reinterpret_cast<PrepSmem *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int chunk = blockIdx.x, h = blockIdx.y;
    if (cu && chunk >= coff[N]) return;

    int seq, len;
    long long t0;
    locate_chunk(chunk, cu, coff, N, T, total_T, cps, seq, t0, len);
    unsigned char *rec = wsp + ((size_t)chunk * H + h) * ws::RECORD;

    // ---- phase 1: g -> smem (zero past the end), beta ----
    for (int i = tid; i < C * (D / 4); i += NT) {
        const int r = i / (D / 4), c4 = i % (D / 4);
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < len) x = *reinterpret_cast<const float4 *>(g + ((size_t)(t0 + r) * H + h) * D + c4 * 4);
        *reinterpret_cast<float4 *>(&sm.G[r][c4 * 4]) = x;
    }
    if (tid < C) sm.beta[tid] = (tid < len) ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
    __syncthreads();

    // ---- phase 2: per-channel cumsum and block tables ----
    if (tid < D) {
        const int c = tid;
        float acc = 0.f;
#pragma unroll 8
        for (int r = 0; r < C; ++r) { acc += sm.G[r][c]; sm.G[r][c] = acc; }
        float R[4];
#pragma unroll
        for (int I = 0; I < 4; ++I) { R[I] = sm.G[16 * I + 15][c]; sm.R[I][c] = R[I]; }
        sm.Eb[0][c] = 1.f;
#pragma unroll
        for (int I = 1; I < 4; ++I) sm.Eb[I][c] = expf(R[I - 1]);
#pragma unroll
        for (int I = 0; I < 3; ++I) sm.F[I][c] = expf(R[3] - R[I]);
        sm.F[3][c] = 1.f;
#pragma unroll
        for (int I = 0; I < 4; ++I)
#pragma unroll
            for (int J = I + 1; J < 4; ++J) sm.Dm[I * 4 + J][c] = expf(R[J - 1] - R[I]);
        reinterpret_cast<float *>(rec + ws::OFF_EGC)[c] = expf(R[3]);
    }
    __syncthreads();

    // ---- phase 3: decayed operand forms (8 channels per item) ----
    for (int it = tid; it < C * (D / 8); it += NT) {
        const int r = it / (D / 8), c0 = (it % (D / 8)) * 8;
        const int I = r >> 4;
        const float br = sm.beta[r];
        uint4 qraw = make_uint4(0, 0, 0, 0), kraw = make_uint4(0, 0, 0, 0);
        if (r < len) {
            const size_t off = ((size_t)(t0 + r) * H + h) * D + c0;
            qraw = *reinterpret_cast<const uint4 *>(q + off);
            kraw = *reinterpret_cast<const uint4 *>(k + off);
        }
        const __nv_bfloat16 *q8 = reinterpret_cast<const __nv_bfloat16 *>(&qraw);
        const __nv_bfloat16 *k8 = reinterpret_cast<const __nv_bfloat16 *>(&kraw);
        uint32_t xk[4], xq[4], kg[4], qg[4], kt[4], krs[4], krv[3][4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            float vxk[2], vxq[2], vkg[2], vqg[2], vkt[2], vkrs[2], vkrv[3][2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int c = c0 + e + u;
                const float G = sm.G[r][c];
                const float Rp = I > 0 ? sm.R[I - 1][c] : 0.f;
                const float a = expf(G - Rp);
                const float b = expf(sm.R[I][c] - G);
                const float kv = __bfloat162float(k8[e + u]);
                const float qv = __bfloat162float(q8[e + u]);
                const float eG = a * sm.Eb[I][c];
                vxk[u] = br * kv * a;
                vxq[u] = qv * a;
                vkg[u] = br * kv * eG;
                vqg[u] = qv * eG;
                vkt[u] = kv * b * sm.F[I][c];
                vkrs[u] = kv / a;
#pragma unroll
                for (int J = 1; J < 4; ++J)
                    vkrv[J - 1][u] = (I + J < 4) ? kv * b * sm.Dm[I * 4 + I + J][c] : 0.f;
            }
            xk[e / 2] = pack_bf16(vxk[0], vxk[1]);
            xq[e / 2] = pack_bf16(vxq[0], vxq[1]);
            kg[e / 2] = pack_bf16(vkg[0], vkg[1]);
            qg[e / 2] = pack_bf16(vqg[0], vqg[1]);
            kt[e / 2] = pack_bf16(vkt[0], vkt[1]);
            krs[e / 2] = pack_bf16(vkrs[0], vkrs[1]);
#pragma unroll
            for (int J = 0; J < 3; ++J) krv[J][e / 2] = pack_bf16(vkrv[J][0], vkrv[J][1]);
        }
        *reinterpret_cast<uint4 *>(&sm.Xk[r][c0]) = make_uint4(xk[0], xk[1], xk[2], xk[3]);
        *reinterpret_cast<uint4 *>(&sm.Xq[r][c0]) = make_uint4(xq[0], xq[1], xq[2], xq[3]);
        *reinterpret_cast<uint4 *>(&sm.KG[r][c0]) = make_uint4(kg[0], kg[1], kg[2], kg[3]);
        // version I holds row r itself (k / a); versions I' > I hold k b Dm
        *reinterpret_cast<uint4 *>(&sm.Kr[kr_base(I) + r][c0]) = make_uint4(krs[0], krs[1], krs[2], krs[3]);
#pragma unroll
        for (int J = 1; J < 4; ++J)
            if (I + J < 4)
                *reinterpret_cast<uint4 *>(&sm.Kr[kr_base(I + J) + r][c0]) =
                    make_uint4(krv[J - 1][0], krv[J - 1][1], krv[J - 1][2], krv[J - 1][3]);
        *reinterpret_cast<uint4 *>(rec + ws::OFF_QG + ((size_t)r * D + c0) * 2) =
            make_uint4(qg[0], qg[1], qg[2], qg[3]);
        *reinterpret_cast<uint4 *>(rec + ws::OFF_KT + ((size_t)r * D + c0) * 2) =
            make_uint4(kt[0], kt[1], kt[2], kt[3]);
    }
    // beta V
    for (int it = tid; it < C * (D / 8); it += NT) {
        const int r = it / (D / 8), c0 = (it % (D / 8)) * 8;
        uint4 vraw = make_uint4(0, 0, 0, 0);
        if (r < len) vraw = *reinterpret_cast<const uint4 *>(v + ((size_t)(t0 + r) * H + h) * D + c0);
        const __nv_bfloat16 *v8 = reinterpret_cast<const __nv_bfloat16 *>(&vraw);
        const float br = sm.beta[r];
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2)
            o[e / 2] = pack_bf16(br * __bfloat162float(v8[e]), br * __bfloat162float(v8[e + 1]));
        *reinterpret_cast<uint4 *>(&sm.Vb[r][c0]) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncthreads();

    // ---- phase 4: A (warps 0-3) and P (warps 4-7), row block I = warp & 3 ----
    {
        const int I = warp & 3;
        const bool isP = warp >= 4;
        const __nv_bfloat16(*X)[PB] = isP ? sm.Xq : sm.Xk;
        float acc[4][2][4];
#pragma unroll
        for (int J = 0; J < 4; ++J)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[J][nt][e] = 0.f;
        const int arow = 16 * I + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int acol = 8 * (lane >> 4);
        const int bn = (lane & 7) + 8 * (lane >> 4);
        const int bk = 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a[4];
            ldsm_x4(a, &X[arow][16 * ks + acol]);
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                if (J <= I) {
                    uint32_t b[4];
                    ldsm_x4(b, &sm.Kr[kr_base(I) + 16 * J + bn][16 * ks + bk]);
                    mma_bf16(acc[J][0], a, b[0], b[1]);
                    mma_bf16(acc[J][1], a, b[2], b[3]);
                }
            }
        }
        __syncthreads();   // G region is now reused as P staging
#pragma unroll
        for (int J = 0; J < 4; ++J)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int i = 16 * I + gid + 8 * hh;
                    const int j = 16 * J + 8 * nt + 2 * tig;
                    float v0 = acc[J][nt][2 * hh], v1 = acc[J][nt][2 * hh + 1];
                    if (!isP) {
                        if (J <= I) {
                            sm.A[i][j] = (j < i) ? v0 : 0.f;
                            sm.A[i][j + 1] = (j + 1 < i) ? v1 : 0.f;
                        }
                    } else {
                        v0 = (J <= I && j <= i) ? v0 : 0.f;
                        v1 = (J <= I && j + 1 <= i) ? v1 : 0.f;
                        *reinterpret_cast<uint32_t *>(&sm.Pst[i][j]) = pack_bf16(v0, v1);
                    }
                }
    }
    __syncthreads();

    // ---- phase 5: T = (I + A)^-1 ----
    if (warp < 4 && lane < 16) {
        const int I = warp, c = lane, o = 16 * I;
        for (int i = 0; i < 16; ++i) {
            float t;
            if (i < c) t = 0.f;
            else if (i == c) t = 1.f;
            else {
                float s = 0.f;
                for (int j = c; j < i; ++j) s += sm.A[o + i][o + j] * sm.Tm[o + j][o + c];
                t = -s;
            }
            sm.Tm[o + i][o + c] = t;
        }
    } else if (warp >= 4) {
        // zero the strictly-upper blocks of T
        const int I = warp - 4;
        for (int e = lane; e < 16 * 64; e += 32) {
            const int i = e / 64, j = e % 64;
            if (j >= 16 * (I + 1)) sm.Tm[16 * I + i][j] = 0.f;
        }
    }
    __syncthreads();
#pragma unroll 1
    for (int dist = 1; dist < 4; ++dist) {
        if (warp < 4 && warp >= dist) {
            const int I = warp, J = I - dist;
            const int i = lane >> 1, c0 = 8 * (lane & 1);
            float z[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) z[e] = 0.f;
            for (int M = J; M < I; ++M)
                for (int m = 0; m < 16; ++m) {
                    const float a = sm.A[16 * I + i][16 * M + m];
#pragma unroll
                    for (int e = 0; e < 8; ++e) z[e] += a * sm.Tm[16 * M + m][16 * J + c0 + e];
                }
#pragma unroll
            for (int e = 0; e < 8; ++e) sm.Zs[warp][i][c0 + e] = z[e];
            __syncwarp();
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float s = 0.f;
                for (int m = 0; m <= i; ++m) s += sm.Tm[16 * I + i][16 * I + m] * sm.Zs[warp][m][c0 + e];
                sm.Tm[16 * I + i][16 * J + c0 + e] = -s;
            }
        }
        __syncthreads();
    }

    // ---- phase 6: W = T (beta K e^G) (warps 0-3), U = T (beta V) (warps 4-7) ----
    {
        const int I = warp & 3;
        const bool isU = warp >= 4;
        const __nv_bfloat16(*B)[PB] = isU ? sm.Vb : sm.KG;
        __nv_bfloat16(*Out)[PB] = isU ? sm.Xq : sm.Xk;
        float acc[16][4];
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
        const int bk = (lane & 7) + 8 * ((lane >> 3) & 1);
        const int bn = 8 * (lane >> 4);
        for (int ks = 0; ks <= I; ++ks) {
            uint32_t a[4];
            const int r0 = 16 * I + gid, k0 = 16 * ks + 2 * tig;
            a[0] = pack_bf16(sm.Tm[r0][k0], sm.Tm[r0][k0 + 1]);
            a[1] = pack_bf16(sm.Tm[r0 + 8][k0], sm.Tm[r0 + 8][k0 + 1]);
            a[2] = pack_bf16(sm.Tm[r0][k0 + 8], sm.Tm[r0][k0 + 9]);
            a[3] = pack_bf16(sm.Tm[r0 + 8][k0 + 8], sm.Tm[r0 + 8][k0 + 9]);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t b[4];
                ldsm_x4_t(b, &B[16 * ks + bk][16 * np + bn]);
                mma_bf16(acc[2 * np], a, b[0], b[1]);
                mma_bf16(acc[2 * np + 1], a, b[2], b[3]);
            }
        }
        __syncthreads();   // Xk/Xq are reused as W/U staging
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            const int i = 16 * I + gid, j = 8 * nt + 2 * tig;
            *reinterpret_cast<uint32_t *>(&Out[i][j]) = pack_bf16(acc[nt][0], acc[nt][1]);
            *reinterpret_cast<uint32_t *>(&Out[i + 8][j]) = pack_bf16(acc[nt][2], acc[nt][3]);
        }
    }
    __syncthreads();

    // ---- phase 7: coalesced record stores ----
    for (int it = tid; it < C * (D / 8); it += NT) {
        const int r = it / (D / 8), c0 = (it % (D / 8)) * 8;
        *reinterpret_cast<uint4 *>(rec + ws::OFF_W + ((size_t)r * D + c0) * 2) =
            *reinterpret_cast<const uint4 *>(&sm.Xk[r][c0]);
        *reinterpret_cast<uint4 *>(rec + ws::OFF_U + ((size_t)r * D + c0) * 2) =
            *reinterpret_cast<const uint4 *>(&sm.Xq[r][c0]);
    }
    for (int it = tid; it < C * (C / 8); it += NT) {
        const int r = it / (C / 8), c0 = (it % (C / 8)) * 8;
        *reinterpret_cast<uint4 *>(rec + ws::OFF_P + ((size_t)r * C + c0) * 2) =
            *reinterpret_cast<const uint4 *>(&sm.Pst[r][c0]);
    }
}

// Chunk offsets per sequence for varlen mode: coff[n] = sum_{m<n} ceil(len_m / C).
__global__ void chunk_plan_kernel(const int32_t *__restrict__ cu, int N, int total_T,
                                  int32_t *__restrict__ coff)
{
    __shared__ int part[1024];
    const int tid = threadIdx.x;
    const int per = (N + 1023) / 1024;
    const int s0 = tid * per, s1 = min(N, s0 + per);
    int sum = 0;
    for (int n = s0; n < s1; ++n) {
        const int b = min(max(cu[n], 0), total_T), e = min(max(cu[n + 1], 0), total_T);
        sum += e > b ? (e - b + C - 1) / C : 0;
    }
    part[tid] = sum;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
        const int x = tid >= off ? part[tid - off] : 0;
        __syncthreads();
        part[tid] += x;
        __syncthreads();
    }
    int run = tid > 0 ? part[tid - 1] : 0;
    for (int n = s0; n < s1; ++n) {
        coff[n] = run;
        const int b = min(max(cu[n], 0), total_T), e = min(max(cu[n + 1], 0), total_T);
        run += e > b ? (e - b + C - 1) / C : 0;
    }
    if (tid == 1023) coff[N] = part[1023];
}

}  // namespace

size_t chunk_prep_smem_bytes() { return sizeof(PrepSmem); }

cudaError_t launch_chunk_plan(const int32_t *cu, int N, int total_T, int32_t *coff,
                              cudaStream_t st)
{
    chunk_plan_kernel<<<1, 1024, 0, st>>>(cu, N, total_T, coff);
    return cudaGetLastError();
}

cudaError_t launch_chunk_prep(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const int32_t *cu, const int32_t *coff,
                              int N, int T, int total_T, int H, int max_chunks,
                              unsigned char *wsp, cudaStream_t st)
{
    const size_t smem = sizeof(PrepSmem);
    cudaError_t e = cudaFuncSetAttribute(chunk_prep_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int cps = (T + C - 1) / C;
    dim3 grid(max_chunks, H);
    chunk_prep_kernel<<<grid, NT, smem, st>>>(
        (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, g, beta,
        cu, coff, N, T, total_T, H, cps, wsp);
    return cudaGetLastError();
}

}  // namespace kda
