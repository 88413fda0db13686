// kda_prefill_tc.cu -- the state passes of the tensor-core KDA prefill
// (sm_100a: tcgen05.mma, TMEM accumulators, bulk copies), bf16 inputs,
// dk = dv = 128, chunk = 64, and the host side of that path.
//
// The chunk preparation (kda_prep_tc.cu) leaves, per (chunk, head), the chain
// operands W, Q', K', A_qk, U~, gamma and 1/|q| in the chunk's slot (Kimi
// Linear summary §3.1: the chunkwise WY / UT form).  What remains is
// sequential over the chunks of a sequence and runs here with the fp32 state
// S [dk x dv] in Tensor Memory (the inter-chunk state carry):
//
//   U = U~ - W S,   O = Q' S + A_qk U,   S <- Diag(gamma) S + K'^T U.
//
// Segments: with P > 1 a sequence is cut into P runs of chunks.  The
// transition pass runs each segment but the last from a zero state and from
// the identity, giving the affine map S_out = M S_in + N of the segment; a
// small kernel composes the maps into every segment's incoming state; the
// full pass then runs every segment from its true incoming state and writes
// the outputs.  This is the single-GPU form of the prefix scan over
// per-segment state updates (Kimi K3 architecture summary, KDA context
// parallelism).
#include <atomic>

#include "kda_tc_common.cuh"

namespace kda {
namespace tcp {
namespace {

// Checkpoint slot of the state after sequence-relative chunk c (n_tok tokens in
// the sequence), or null when no checkpoint falls there.
__device__ __forceinline__ float* ckpt_state(const TcParams& p, int n, int h, int c, int n_tok) {
  if (!p.S_ckpt || (c + 1) % p.ckpt_every != 0 || (c + 1) * 64 > n_tok) return nullptr;
  return p.S_ckpt + (((size_t)n * p.H + h) * p.ckpt_count + (c + 1) / p.ckpt_every - 1) * 128 * 128;
}

// ---------------------------------------------------------------------------
// Chain passes: the state-dependent half of each chunk, from the operands in
// its slot.  The state is kept transposed in Tensor Memory, S^T with the value
// column as the lane and the key channel as the column (fp32, 128 x 128), so
// that both A operands of the chain, an f16 copy of S^T and U^T, are read by
// the MMAs from Tensor Memory and only the slot's images come from shared
// memory.  Per chunk:
//   C1: [D_Q^T | D_W^T] = S^T [Q' ; W]^T   (M=128 value columns, N=128 tokens);
//   U^T = U~^T - D_W^T  (f16, in Tensor Memory);
//   C2: S^T += U^T K'  (M=128, N=128 key channels) and D_Q^T += U^T A_qk^T
//       (N=64), one N=192 product in the full pass;
//   the new S^T is copied to f16 for the next C1 and, in place, scaled by the
//   next chunk's gamma (per key channel) before that chunk's C2 accumulates
//   into it; o = (D_Q^T)^T / |q| of a chunk is written during the next C1.
//   TRANS = false: full pass of segment p from its true incoming state; o, S_final.
//   TRANS = true : transition of segments 0..P-2 on [S | X] from S = 0 (-> N_p)
//                  and X = I (-> M_p), X^T a second 128-lane block; no Q', no o.
// Slot parts are bulk-copied ahead into a ring of stages (three chunks ahead in
// the full pass, four in the transition pass, whose stages are smaller).
template <bool TRANS>
struct ChainSmem {
  static constexpr int kStages = TRANS ? 4 : 3;
  // stage layout: the slot (full pass), or W | K' | U~^T | gamma (transition: the
  // W half of the [Q' ; W] image; no Q', A_qk or 1/|q|; one bulk copy per part)
  static constexpr int kK = TRANS ? 16384 : kSlotK;
  static constexpr int kUt = TRANS ? 32768 : kSlotU;
  static constexpr int kGam = TRANS ? 32768 + 16384 : kSlotGam;
  static constexpr int kStageBytes = TRANS ? 32768 + 16384 + 512 : kSlotBytes;
  static constexpr int kBytes = kStages * kStageBytes;
};
// TMEM columns (512 allocated): fp32 S^T, fp32 X^T (transition), the products D^T
// (full pass: [D_Q^T | D_W^T] right after S^T, so that C2 accumulates into
// [S^T | D_Q^T] with one N = 192 product per K step; transition: D_S^T | D_X^T),
// and the f16 copies of S^T (and X^T), whose columns hold U^T while C2 runs.
template <bool TRANS>
struct ChainTmem {
  static constexpr uint32_t kS = 0, kX = 128;
  static constexpr uint32_t kD0 = TRANS ? 256 : 128;  // the products of C1
  static constexpr uint32_t kDQ = 128, kDW = 192;     // full pass: D_Q^T, D_W^T
  static constexpr uint32_t kCp = 384;  // S^T copy (64 columns), then X^T copy
};

template <bool TRANS>
__global__ void __launch_bounds__(kNT, 1) chain_kernel(const __grid_constant__ TcParams p) {
  using L = ChainSmem<TRANS>;
  using TM = ChainTmem<TRANS>;
  constexpr int NB = TRANS ? 2 : 1;  // 128-lane state blocks: S^T, and X^T
  constexpr int NS = L::kStages;
  extern __shared__ __align__(1024) unsigned char sm[];
  __shared__ uint64_t s_bar, s_ld[NS];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ float s_iq[64];        // 1/|q| of the chunk whose o is written next
  __shared__ float s_red[4][64];    // output epilogue: sum of squares per lane quarter and token
  __shared__ float s_rs[64];        // output epilogue: 1 / RMS of each token's o row

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x, h = blockIdx.y, seg = blockIdx.z;
  const int H = p.H;
  if (!seqlens_valid(p.cu, p.N, p.T, p.max_len)) return;  // the error word is already set
  int a, b;
  seq_bounds(p.cu, n, p.max_len, a, b);
  const int nch = (b - a + kC - 1) / kC;
  int c0, c1;
  segment_chunks(nch, p.P, seg, c0, c1);

  if (warp == 0) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&s_bar, 1);
#pragma unroll
    for (int s = 0; s < NS; ++s) mbar_init(&s_ld[s], 1);
    fence_mbar_init();
    s_abort = 0;
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = s_tmem;
  auto stage_of = [&](int c) { return (c - c0) % NS; };
  auto load_slot = [&](int c) {  // single thread
    const int s = stage_of(c);
    unsigned char* dst = sm + s * L::kStageBytes;
    const unsigned char* src = chunk_slot(p.prep, a, n, c, h, H);
    mbar_arrive_expect_tx(&s_ld[s], L::kStageBytes);
    if (TRANS) {
      bulk_g2s(dst, src + kSlotWQ + 16384, 16384, &s_ld[s]);             // W
      bulk_g2s(dst + L::kK, src + kSlotK, 16384, &s_ld[s]);             // K'
      bulk_g2s(dst + L::kUt, src + kSlotU, 16384 + 512, &s_ld[s]);      // U~^T | gamma
    } else {
      bulk_g2s(dst, src, kSlotBytes, &s_ld[s]);
    }
  };
  if (tid == 0)
    for (int c = c0; c < c1 && c < c0 + NS; ++c) load_slot(c);
  uint32_t phase = 0, ph_ld = 0;  // ph_ld bit s: parity of stage s's next completion
  bool mma_pending = false;       // products committed and not yet awaited
  uint32_t inflight = 0;          // stages being filled
  for (int c = c0; c < c1 && c < c0 + NS; ++c) inflight |= 1u << stage_of(c);
  // Block-wide bounded wait for the stage of chunk c; false if it gave up.
  auto wait_stage = [&](int c) -> bool {
    const int s = stage_of(c);
    const bool got = mbar_wait_cycles(&s_ld[s], (ph_ld >> s) & 1, p.wait_limit);
    if (__syncthreads_or(!got)) {
      if (tid == 0) atomicOr(&p.hdr->err, kErrTimeout);
      return false;
    }
    ph_ld ^= 1u << s;
    inflight &= ~(1u << s);
    return true;
  };

  const int q4 = warp & 3, cq = warp >> 2;  // TMEM lane quarter, column quarter
  const int v = 32 * q4 + lane;             // TMEM lane: value column of S^T / D^T, column of X^T
  const uint32_t lq = (uint32_t)(32 * q4) << 16;  // this warp's lane quarter in a TMEM address

  // f16 copy of 32 fp32 state columns (key channels 32 cq ..) into the A-operand image
  auto put_copy = [&](uint32_t col, const float* s32) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = h2(s32[2 * i], s32[2 * i + 1]);
    tmem_st16u(tm + lq + col, w);
  };

  // ---- initial state -> TMEM: S^T[v][k] = S_in[k][v] (full pass), or S = 0 and
  //      X^T = I (transition)
  {
    const float* S0 = nullptr;
    if (!TRANS)
      S0 = seg > 0 ? seg_sin(p.seg, n, h, H, p.Pseg, seg)
                   : (p.S0 ? p.S0 + ((size_t)n * H + h) * kD * kD : nullptr);
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      float s32[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int k = 32 * cq + i;
        s32[i] = S0 ? S0[(size_t)k * kD + v] : (blk == 1 && k == v) ? 1.f : 0.f;
      }
      tmem_st16(tm + lq + TM::kS + 128 * blk + 32 * cq, *reinterpret_cast<float(*)[16]>(s32));
      tmem_st16(tm + lq + TM::kS + 128 * blk + 32 * cq + 16, *reinterpret_cast<float(*)[16]>(s32 + 16));
      put_copy(TM::kCp + 64 * blk + 16 * cq, s32);
    }
    tmem_st_wait();
  }

  // ---- o of a chunk from D_Q^T: lane v holds its column for tokens 16 cq ..
  //      16 cq + 15, loaded into x by load_o before the next chunk's C1
  //      overwrites the product columns; with the output epilogue the sums of
  //      squares over the 128 columns meet in shared memory.
  // Output epilogue: the gate inputs of chunk cc (raw bf16 bits in rgr) are
  // requested a chunk ahead, while the previous chunk's C2 product runs, and
  // not touched until they are turned into sigmoids (sg) while cc's own C2
  // runs, so their latency stays off the chain's critical path; write_o(cc)
  // uses sg during the next chunk's C1.
  uint32_t rgr[16];
  float sg[16];
  const float wv = (p.og && p.ow) ? p.ow[v] : 1.f;
  auto load_gate = [&](int cc) {
    if (!p.og) return;
    const int t0c = a + cc * kC, lenc = min(kC, b - t0c);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int t = 16 * cq + i;
      rgr[i] = t < lenc ? *reinterpret_cast<const uint16_t*>(p.og + ((size_t)(t0c + t) * H + h) * kD + v) : 0u;
    }
  };
  auto gate_sigmoids = [&]() {
    if (!p.og) return;
#pragma unroll
    for (int i = 0; i < 16; ++i) sg[i] = out_sigmoid(__uint_as_float(rgr[i] << 16));
  };
  auto load_o = [&](float (&x)[16]) {
    tmem_ld16(tm + lq + TM::kDQ + 16 * cq, x);
    tmem_ld_wait();
  };
  auto write_o = [&](int cc, float (&x)[16]) {
    const int t0c = a + cc * kC, lenc = min(kC, b - t0c);
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] *= s_iq[16 * cq + i];
    if (p.og) {
      // sums of squares over this warp's 32 columns for each of its 16 tokens:
      // a butterfly that halves the token count per step leaves token
      // (lane >> 1) & 15 on each lane
      float y[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) y[i] = x[i] * x[i];
#pragma unroll
      for (int st = 8; st >= 1; st >>= 1) {
        const bool up = (lane & (2 * st)) != 0;  // keep the upper half of the tokens
#pragma unroll
        for (int i = 0; i < st; ++i) {
          const float send = up ? y[i] : y[i + st];
          const float keep = up ? y[i + st] : y[i];
          y[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2 * st);
        }
      }
      y[0] += __shfl_xor_sync(0xffffffffu, y[0], 1);
      // lane l holds token t = (bit 4 of l) * 8 + (bit 3) * 4 + (bit 2) * 2 + (bit 1)
      const int tl = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
      if ((lane & 1) == 0) s_red[q4][16 * cq + tl] = y[0];
      asm volatile("bar.sync %0, 128;" ::"r"(1 + cq) : "memory");  // the four warps of column quarter cq
      if (q4 == 0 && lane < 16) {  // one reciprocal RMS per token
        const int t = 16 * cq + lane;
        s_rs[t] = rsqrtf((s_red[0][t] + s_red[1][t] + s_red[2][t] + s_red[3][t]) * (1.0f / kD) + p.oeps);
      }
      asm volatile("bar.sync %0, 128;" ::"r"(1 + cq) : "memory");  // s_rs is written
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] = x[i] * s_rs[16 * cq + i] * (wv * sg[i]);
    }
    // lanes v and v ^ 1 swap halves so that each stores bf16 pairs of adjacent columns
    const bool odd = lane & 1;
    const int vb = v & ~1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float mine_lo = odd ? x[8 + i] : x[i];        // the token this lane stores
      const float give = odd ? x[i] : x[8 + i];           // the partner's token
      const float other = __shfl_xor_sync(0xffffffffu, give, 1);
      const int t = 16 * cq + (odd ? 8 + i : i);
      const float lo = odd ? other : mine_lo, hi = odd ? mine_lo : other;
      if (t < lenc) {
        __nv_bfloat162 pr = __floats2bfloat162_rn(lo, hi);
        *reinterpret_cast<__nv_bfloat162*>(p.o + ((size_t)(t0c + t) * H + h) * kD + vb) = pr;
      }
    }
  };
  // fp32 state (and X^T) columns times gamma of the key channel, in TMEM
  auto decay_state = [&](const float* gam) {
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      float s0[16], s1[16];
      const uint32_t col = TM::kS + 128 * blk + 32 * cq;
      tmem_ld16(tm + lq + col, s0);
      tmem_ld16(tm + lq + col + 16, s1);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) { s0[i] *= gam[32 * cq + i]; s1[i] *= gam[32 * cq + 16 + i]; }
      tmem_st16(tm + lq + col, s0);
      tmem_st16(tm + lq + col + 16, s1);
    }
    tmem_st_wait();
  };

  // the first chunk's stage; later stages are awaited at the end of the chunk before
  if (!TRANS && c0 < c1) load_gate(c0);
  if (c0 < c1 && !wait_stage(c0)) s_abort = 1;
  for (int c = c0; c < c1 && !s_abort; ++c) {
    const int s = stage_of(c);
    unsigned char* st = sm + s * L::kStageBytes;
    // the previous chunk's D_Q^T leaves the product columns before C1 reuses them
    float xo[16];
    if (!TRANS && c > c0) load_o(xo);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    // ---- C1: A = the f16 copy of S^T (X^T) in TMEM; B = [Q' ; W] or W, MN-major
    if (tid == 0) {
      if (!TRANS) {
        constexpr uint32_t id = instr_desc(kFmtF16, 128, 128, false, true);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t bd = smem_desc(smem_u32(st + kSlotWQ + k * 256), 128, 2048);
          mma_f16_ts(tm + TM::kD0, tm + TM::kCp + 8 * k, bd, id, k > 0);
        }
      } else {
        constexpr uint32_t id = instr_desc(kFmtF16, 128, 64, false, true);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t bd = smem_desc(smem_u32(st + k * 256), 128, 2048);  // W
          mma_f16_ts(tm + TM::kD0, tm + TM::kCp + 8 * k, bd, id, k > 0);
          mma_f16_ts(tm + TM::kD0 + 64, tm + TM::kCp + 64 + 8 * k, bd, id, k > 0);
        }
      }
      mma_commit(&s_bar);
    }
    mma_pending = true;
    // ---- meanwhile: the first chunk decays the incoming state by its gamma (later
    //      chunks get it with the previous chunk's copy); the previous o goes out
    if (c == c0) decay_state(reinterpret_cast<const float*>(st + L::kGam));
    if (!TRANS && c > c0) write_o(c - 1, xo);
    if (!block_wait(&s_bar, phase, p.hdr, p.wait_limit)) { s_abort = 1; break; }
    mma_pending = false;
    // ---- U^T = U~^T - D_W^T (transition: U_S^T = U~^T - D_S^T, U_X^T = -D_X^T),
    //      f16 into the copy's columns (C1 has read them)
    {
      float d[16];
      tmem_ld16(tm + lq + (TRANS ? TM::kD0 : TM::kDW) + 16 * cq, d);
      float dx[16];
      if (TRANS) tmem_ld16(tm + lq + TM::kD0 + 64 + 16 * cq, dx);
      const uint4* ug = reinterpret_cast<const uint4*>(st + L::kUt);
      float u[16];
      unpack8h(ug[ut_index(q4, cq, 0, lane)], u);
      unpack8h(ug[ut_index(q4, cq, 1, lane)], u + 8);
      tmem_ld_wait();
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = h2(u[2 * i] - d[2 * i], u[2 * i + 1] - d[2 * i + 1]);
      tmem_st8(tm + lq + TM::kCp + 8 * cq, w);
      if (TRANS) {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = h2(-dx[2 * i], -dx[2 * i + 1]);
        tmem_st8(tm + lq + TM::kCp + 64 + 8 * cq, w);
      }
      tmem_st_wait();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    // ---- C2: S^T (X^T) += U^T K' (B = K' K-major: N = key channel, K = token);
    //      full pass: with D_Q^T += U^T A_qk^T in the same product, B = [K' | A_qk^T]
    //      (N = 128 key channels, then 64 query rows; K = key row)
    if (tid == 0) {
      constexpr uint32_t id = instr_desc(kFmtF16, 128, TRANS ? 128 : 192, false, false);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t kd = smem_desc(smem_u32(st + L::kK + k * 256), 128, 1024);
        mma_f16_ts(tm + TM::kS, tm + TM::kCp + 8 * k, kd, id, 1);
        if (TRANS) mma_f16_ts(tm + TM::kX, tm + TM::kCp + 64 + 8 * k, kd, id, 1);
      }
      mma_commit(&s_bar);
    }
    mma_pending = true;
    // the query row scales of this chunk, for its o (written during the next C1)
    if (!TRANS && tid < kC) s_iq[tid] = reinterpret_cast<const float*>(st + kSlotIq)[tid];
    if (!TRANS) {
      gate_sigmoids();                  // this chunk's epilogue gates, while C2 runs
      if (c + 1 < c1) load_gate(c + 1);  // and the next chunk's inputs
    }
    if (!block_wait(&s_bar, phase, p.hdr, p.wait_limit)) { s_abort = 1; break; }
    mma_pending = false;
    // the stage is consumed (its reads ended before the barrier above): refill it
    if (c + NS < c1) {
      inflight |= 1u << s;
      if (tid == 0) load_slot(c + NS);
    }
    // the next chunk's stage, for its gamma
    if (c + 1 < c1 && !wait_stage(c + 1)) { s_abort = 1; break; }
    const float* gnext =
        c + 1 < c1 ? reinterpret_cast<const float*>(sm + stage_of(c + 1) * L::kStageBytes + L::kGam)
                   : nullptr;
    // ---- S^T (X^T) -> f16 copy for the next chunk (and the fp32 checkpoint, if one
    //      falls after this chunk); the TMEM state takes the next chunk's decay
    float* ck = TRANS ? nullptr : ckpt_state(p, n, h, c, b - a);
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      float s32[32];
      const uint32_t col = TM::kS + 128 * blk + 32 * cq;
      tmem_ld16(tm + lq + col, *reinterpret_cast<float(*)[16]>(s32));
      tmem_ld16(tm + lq + col + 16, *reinterpret_cast<float(*)[16]>(s32 + 16));
      tmem_ld_wait();
      if (ck) {
#pragma unroll
        for (int i = 0; i < 32; ++i) ck[(size_t)(32 * cq + i) * kD + v] = s32[i];
      }
      put_copy(TM::kCp + 64 * blk + 16 * cq, s32);
      if (gnext) {
#pragma unroll
        for (int i = 0; i < 32; ++i) s32[i] *= gnext[32 * cq + i];
        tmem_st16(tm + lq + col, *reinterpret_cast<float(*)[16]>(s32));
        tmem_st16(tm + lq + col + 16, *reinterpret_cast<float(*)[16]>(s32 + 16));
      }
    }
    tmem_st_wait();
  }
  // o of the last chunk
  if (!TRANS && !s_abort && c1 > c0) {
    __syncthreads();  // s_iq of the last chunk (its gate sigmoids are in sg)
    float xo[16];
    load_o(xo);
    write_o(c1 - 1, xo);
  }

  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (!s_abort) {
    float* dst0 = nullptr;
    if (TRANS)
      dst0 = seg_trans(p.seg, n, h, H, p.Pseg, seg);  // M_p, then N_p
    else if (p.S_final && seg == p.P - 1)
      dst0 = p.S_final + ((size_t)n * H + h) * kD * kD;
    if (dst0) {
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        float s32[32];
        tmem_ld16(tm + lq + TM::kS + 128 * blk + 32 * cq, *reinterpret_cast<float(*)[16]>(s32));
        tmem_ld16(tm + lq + TM::kS + 128 * blk + 32 * cq + 16, *reinterpret_cast<float(*)[16]>(s32 + 16));
        tmem_ld_wait();
        // transition: S (block 0) is N_p, X (block 1) is M_p; both stored [key][column]
        float* dst = TRANS ? dst0 + (blk == 0 ? kD * kD : 0) : dst0;
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[(size_t)(32 * cq + i) * kD + v] = s32[i];
      }
    }
  } else if (tid == 0) {
    // a wait gave up: let the slot copies and products still in flight land
    // before the CTA frees its Tensor Memory and leaves (at most ~2 s each)
    for (int s = 0; s < NS; ++s)
      if (inflight & (1u << s)) (void)mbar_wait_cycles(&s_ld[s], (ph_ld >> s) & 1, kWaitCycles);
    if (mma_pending) (void)mbar_wait_cycles(&s_bar, phase, kWaitCycles);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 512);
}

// Incoming state of every segment: S_in(0) = S0, S_in(p+1) = M_p S_in(p) + N_p.
// One CTA per (n, h, 16-column block of the state); fp32 on CUDA cores.  Each
// M_p (64 KB) is bulk-copied into shared memory one step ahead.  The product
// splits the contraction over lanes: warp (column group cg, row half rh) owns
// columns 4 cg .. 4 cg + 3 and rows 64 rh .. 64 rh + 63; lane (row set rs, key
// part kp) keeps the state at keys 4 kp + 32 j + e (j, e < 4) of its four
// columns in registers, reads those keys of its 16 rows of M_p as float4 (one
// 128-byte row segment per 8 lanes), and the 8 partial sums of each output
// meet by shuffles.  The state columns are kept transposed in shared memory.
constexpr int kComposeThreads = 256;
constexpr int kSct = kD + 4;  // row stride (floats) of the transposed state columns
struct ComposeSmem {
  static constexpr int kM = 0;                        // two M_p buffers, [128][128] fp32
  static constexpr int kS = 2 * kD * kD * 4;          // state columns, [16][kSct] fp32
  static constexpr int kBar = kS + 16 * kSct * 4;     // two mbarriers
  static constexpr int kBytes = kBar + 16;
};

// FOLD = false: incoming states S_in(p + 1) = M_p S_in(p) + N_p of segments
// 1 .. P-1 from S_in(0) = S0 (16 state columns per CTA).
// FOLD = true: the transition of the whole sequence, [N | M] = fold over all
// P segments of [N | M] <- M_p [N | M] + [N_p | 0] from [0 | I], written to
// N_out and M_out (16 of the 256 columns of [N | M] per CTA).
template <bool FOLD>
__global__ void __launch_bounds__(kComposeThreads) compose_kernel(const __grid_constant__ TcParams p) {
  using L = ComposeSmem;
  extern __shared__ __align__(1024) unsigned char sm[];
  const int n = blockIdx.x, h = blockIdx.y, cb = blockIdx.z * 16;
  const int H = p.H, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (!seqlens_valid(p.cu, p.N, p.T, p.max_len)) return;
  float* Sct = reinterpret_cast<float*>(sm + L::kS);  // Sct[cc][r] = S[r][cb + cc]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::kBar);
  const int steps = FOLD ? p.P : p.P - 1;
  const bool addn = !FOLD || cb < kD;  // columns of N take N_p; columns of M do not
  auto load_m = [&](int sg) {  // single thread
    mbar_arrive_expect_tx(&bar[sg & 1], kD * kD * 4);
    bulk_g2s(sm + L::kM + (sg & 1) * kD * kD * 4, seg_trans(p.seg, n, h, H, p.Pseg, sg), kD * kD * 4,
             &bar[sg & 1]);
  };
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0 && steps > 0) load_m(0);
  for (int e = tid; e < kD * 16; e += kComposeThreads) {
    const int r = e >> 4, cc = e & 15;
    if (FOLD)
      Sct[cc * kSct + r] = (cb >= kD && r == cb - kD + cc) ? 1.f : 0.f;
    else
      Sct[cc * kSct + r] = p.S0 ? p.S0[((size_t)n * H + h) * kD * kD + (size_t)r * kD + cb + cc] : 0.f;
  }
  // this lane's part of the product
  const int cg = warp & 3, rh = warp >> 2, kp = lane & 7, rs = lane >> 3;
  const int b2 = (lane >> 2) & 1, b1 = (lane >> 1) & 1;
  const int ci = 2 * b2 + b1;            // the column (of cg's four) this lane ends with
  const int col = 4 * cg + ci;           // ... of the CTA's 16
  const int rbase = 64 * rh + 16 * rs;   // its rows: rbase .. rbase + 15
  const bool writer = (lane & 1) == 0;   // lanes 2m and 2m + 1 end with the same sum
  uint32_t inflight = steps > 0 ? 1u : 0u;  // buffers being filled
  uint32_t ph = 0;                            // bit b: parity of buffer b's next completion
  bool ok = true;
  __syncthreads();
  for (int sg = 0; sg < steps; ++sg) {
    const int buf = sg & 1;
    // M_{sg+1} into the other buffer (its readers finished before the last barrier)
    if (sg + 1 < steps) {
      if (tid == 0) load_m(sg + 1);
      inflight |= 1u << (buf ^ 1);
    }
    // N_p of this lane's outputs: issued now, added after the product
    float nv[16];
    {
      const float* Nt = seg_trans(p.seg, n, h, H, p.Pseg, sg) + kD * kD;
#pragma unroll
      for (int i = 0; i < 16; ++i) nv[i] = addn ? Nt[(size_t)(rbase + i) * kD + cb + col] : 0.f;
    }
    // the state at this lane's keys and columns
    float sv[4][16];
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 x = *reinterpret_cast<const float4*>(Sct + (4 * cg + c4) * kSct + 4 * kp + 32 * j);
        sv[c4][4 * j] = x.x;
        sv[c4][4 * j + 1] = x.y;
        sv[c4][4 * j + 2] = x.z;
        sv[c4][4 * j + 3] = x.w;
      }
    const bool got = mbar_wait_cycles(&bar[buf], (ph >> buf) & 1, p.wait_limit);
    if (__syncthreads_or(!got)) {
      if (tid == 0) atomicOr(&p.hdr->err, kErrTimeout);
      ok = false;
      break;
    }
    ph ^= 1u << buf;
    inflight &= ~(1u << buf);
    const float* Ms = reinterpret_cast<const float*>(sm + L::kM + buf * kD * kD * 4);
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float* mr = Ms + (rbase + i) * kD + 4 * kp;
      float pc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 m4 = *reinterpret_cast<const float4*>(mr + 32 * j);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          pc[c4] = fmaf(m4.x, sv[c4][4 * j],
                        fmaf(m4.y, sv[c4][4 * j + 1],
                             fmaf(m4.z, sv[c4][4 * j + 2], fmaf(m4.w, sv[c4][4 * j + 3], pc[c4]))));
      }
      // the sums over the 8 key parts (lane bits 0..2): bit 2 splits the columns
      // into pairs, bit 1 into single columns, bit 0 completes the sum
      const float k0 = b2 ? pc[2] : pc[0], s0 = b2 ? pc[0] : pc[2];
      const float k1 = b2 ? pc[3] : pc[1], s1 = b2 ? pc[1] : pc[3];
      const float q0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 4);
      const float q1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 4);
      float r1 = (b1 ? q1 : q0) + __shfl_xor_sync(0xffffffffu, b1 ? q0 : q1, 2);
      r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
      acc[i] = r1;
    }
    __syncthreads();  // every lane has read the state columns and this M_p
    if (writer) {
#pragma unroll
      for (int i = 0; i < 16; ++i) Sct[col * kSct + rbase + i] = acc[i] + nv[i];
    }
    __syncthreads();
    if (!FOLD) {
      float* Sin = seg_sin(p.seg, n, h, H, p.Pseg, sg + 1);
      for (int e = tid; e < kD * 16; e += kComposeThreads) {
        const int r = e >> 4, cc = e & 15;
        Sin[(size_t)r * kD + cb + cc] = Sct[cc * kSct + r];
      }
    }
  }
  if (FOLD && ok) {
    float* dst = (cb < kD ? p.N_out + cb : p.M_out + (cb - kD)) + ((size_t)n * H + h) * kD * kD;
    for (int e = tid; e < kD * 16; e += kComposeThreads) {
      const int r = e >> 4, cc = e & 15;
      dst[(size_t)r * kD + cc] = Sct[cc * kSct + r];
    }
  }
  if (!ok && tid == 0) {
    // a wait gave up: let the copies still in flight land before leaving
    for (int b2w = 0; b2w < 2; ++b2w)
      if (inflight & (1u << b2w)) (void)mbar_wait_cycles(&bar[b2w], (ph >> b2w) & 1, kWaitCycles);
  }
}


// cuTensorMapEncodeTiled from the driver, looked up once (no link to libcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

// [T, H, 128] bf16 tensor; box `rows` tokens x 1 head x 64 channels with the
// 128-byte swizzle; rows before 0 or past T read as zero.
bool make_map(CUtensorMap* map, const void* base, int T, int H, int rows = kC) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
  const cuuint32_t box[3] = {(cuuint32_t)(kD / 2), 1, (cuuint32_t)rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace tcp

using namespace tcp;

bool tc_supported(const ForwardArgs& a) {
  return a.bf16 && a.dk == kD && a.dv == kD && a.chunk == kC;
}

int tc_segments(int N, int H, int max_len) {
  // enough (sequence, head, segment) CTAs to fill the 148 SMs; long sequences only
  if (N <= 0 || H <= 0) return 1;
  const long long pairs = (long long)N * H;
  int P = pairs >= 128 ? 1 : (int)(148 / pairs);
  const int nch = (max_len + kC - 1) / kC;
  if (P > nch / 2) P = nch / 2;
  if (P < 1) P = 1;
  if (P > 16) P = 16;
  return P;
}

// Workspace: header | per (n, h) segment transitions and incoming states |
// one chain-operand slot per (chunk, head), 1 KB aligned.
static size_t seg_bytes(int N, int H, int P) {
  const size_t per = (size_t)(P - 1) * 2 * kD * kD + (size_t)P * kD * kD;
  return sizeof(WsHeader) + (size_t)N * H * per * sizeof(float);
}
static size_t prep_offset(int N, int H, int P) { return (seg_bytes(N, H, P) + 1023) & ~(size_t)1023; }

size_t tc_workspace_bytes(int N, int T, int H, int max_len) {
  const int P = tc_segments(N, H, max_len);
  const size_t slots = (size_t)T / kC + (size_t)N;
  return prep_offset(N, H, P) + slots * H * kSlotBytes;
}

int tc_launches(int N, int H, int max_len) {
  if (N <= 0) return 0;
  return tc_segments(N, H, max_len) > 1 ? 4 : 2;
}

namespace {

// Limit of the first-giving-up waits of the tensor-core kernels (SM cycles);
// kda_debug_set_wait_limit lowers it to exercise the timeout path.
std::atomic<long long> g_wait_limit{kWaitCycles};

// Kernel parameters of a call; tensor maps only when the call stages inputs.
cudaError_t fill_params(const ForwardArgs& a, TcParams& p, bool maps) {
  memset(&p, 0, sizeof(p));
  if (maps && a.T > 0) {
    const void* zz = a.z ? a.z : a.k;
    const int rows = a.conv_width > 0 ? kC + 8 : kC;  // with the convolution's history
    if (!make_map(&p.sq, a.q, a.T, a.H, rows) || !make_map(&p.sk, a.k, a.T, a.H, rows) ||
        !make_map(&p.sz, zz, a.T, a.H) || !make_map(&p.sv, a.v, a.T, a.H, rows))
      return cudaErrorInvalidValue;
  }
  p.beta = (const __nv_bfloat16*)a.beta;
  p.q = (const __nv_bfloat16*)a.q;
  p.k = (const __nv_bfloat16*)a.k;
  p.z = (const __nv_bfloat16*)a.z;
  p.v = (const __nv_bfloat16*)a.v;
  p.A = a.A;
  p.g = a.g_head ? a.g_head : a.g;
  p.S0 = a.S0;
  p.cu = a.cu;
  p.o = (__nv_bfloat16*)a.o;
  p.S_final = a.S_final;
  p.S_ckpt = a.S_ckpt;
  p.ckpt_every = a.ckpt_every;
  p.ckpt_count = a.ckpt_count;
  p.og = (const __nv_bfloat16*)a.out_gate;
  p.ow = a.norm_w;
  p.oeps = a.norm_eps;
  p.N = a.N;
  p.T = a.T;
  p.max_len = a.max_len;
  p.H = a.H;
  p.P = tc_segments(a.N, a.H, a.max_len);
  p.Pseg = p.P;
  p.hdr = (WsHeader*)a.ws;
  p.seg = (float*)((char*)a.ws + sizeof(WsHeader));
  p.wait_limit = g_wait_limit.load();
  p.cwq = a.conv_wq;
  p.cwk = a.conv_wk;
  p.cwv = a.conv_wv;
  p.cw = a.conv_width;
  return cudaSuccess;
}

int gate_src(const ForwardArgs& a) {
  return a.g_head ? kGateHead : a.g ? kGateChannel : kGateZ;
}

template <bool TRANS>
cudaError_t launch_chain(const TcParams& p, int segments, cudaStream_t st) {
  cudaError_t err = cudaFuncSetAttribute(chain_kernel<TRANS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         ChainSmem<TRANS>::kBytes);
  if (err != cudaSuccess) return err;
  chain_kernel<TRANS><<<dim3(p.N, p.H, segments), kNT, ChainSmem<TRANS>::kBytes, st>>>(p);
  return cudaGetLastError();
}

template <bool FOLD>
cudaError_t launch_compose(const TcParams& p, cudaStream_t st) {
  cudaError_t err = cudaFuncSetAttribute(compose_kernel<FOLD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         ComposeSmem::kBytes);
  if (err != cudaSuccess) return err;
  const int blocks = (FOLD ? 2 * kD : kD) / 16;
  compose_kernel<FOLD><<<dim3(p.N, p.H, blocks), kComposeThreads, ComposeSmem::kBytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward_tc(const ForwardArgs& a) {
  TcParams p;
  cudaError_t err = fill_params(a, p, true);
  if (err != cudaSuccess) return err;
  // chunk preparation -> (segment transitions -> incoming states ->) chain pass
  p.prep = (unsigned char*)a.ws + prep_offset(a.N, a.H, p.Pseg);
  if ((err = launch_prep_tc(p, gate_src(a), a.stream)) != cudaSuccess) return err;
  if (p.P > 1) {
    if ((err = launch_chain<true>(p, p.P - 1, a.stream)) != cudaSuccess) return err;
    if ((err = launch_compose<false>(p, a.stream)) != cudaSuccess) return err;
  }
  return launch_chain<false>(p, p.P, a.stream);
}

void tc_set_wait_limit(long long cycles) { g_wait_limit.store(cycles > 0 ? cycles : kWaitCycles); }

// Context parallelism.  The workspace holds the segment buffers for P + 1
// segments (room for all P transitions) and the chunk slots, and it carries
// the slots and transitions from the local pass to the finishing pass.
size_t tc_cp_workspace_bytes(int N, int T, int H, int max_len) {
  const int P = tc_segments(N, H, max_len);
  const size_t slots = (size_t)T / kC + (size_t)N;
  return prep_offset(N, H, P + 1) + slots * H * kSlotBytes;
}

int tc_cp_local_launches() { return 3; }
int tc_cp_finish_launches(int N, int H, int max_len) {
  return tc_segments(N, H, max_len) > 1 ? 2 : 1;
}

cudaError_t launch_cp_local_tc(const ForwardArgs& a, float* M_out, float* N_out) {
  TcParams p;
  cudaError_t err = fill_params(a, p, true);
  if (err != cudaSuccess) return err;
  p.Pseg = p.P + 1;
  p.prep = (unsigned char*)a.ws + prep_offset(a.N, a.H, p.Pseg);
  p.M_out = M_out;
  p.N_out = N_out;
  if ((err = launch_prep_tc(p, gate_src(a), a.stream)) != cudaSuccess) return err;
  if ((err = launch_chain<true>(p, p.P, a.stream)) != cudaSuccess) return err;
  return launch_compose<true>(p, a.stream);
}

cudaError_t launch_cp_finish_tc(const ForwardArgs& a) {
  TcParams p;
  cudaError_t err = fill_params(a, p, false);
  if (err != cudaSuccess) return err;
  p.Pseg = p.P + 1;
  p.prep = (unsigned char*)a.ws + prep_offset(a.N, a.H, p.Pseg);
  if (p.P > 1 && (err = launch_compose<false>(p, a.stream)) != cudaSuccess) return err;
  return launch_chain<false>(p, p.P, a.stream);
}

}  // namespace kda
