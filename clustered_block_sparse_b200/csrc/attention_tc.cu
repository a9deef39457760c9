// Block-sparse attention with linear compensation on the sm_100a tensor cores
// (SVG-EAR §4.1 routing mask, §4.3 Linear Compensation), bf16 inputs, fp32
// accumulation.
//
// One CTA = one unit of up to 256 permuted query rows of ONE query cluster a,
// split in two 128-row tiles A and B (tcgen05.mma M = 128).  Both tiles walk
// the same key chunks.  A chunk is up to two 32-row boxes (64 keys):
//   * exact boxes: the rows of every key cluster b listed for a, 32 at a
//     time (the last box of a cluster is partial), so small clusters share
//     a chunk instead of each paying for a whole MMA round;
//   * compensation chunks (EAR_COMPENSATE): the C_k key / value centroids, 32
//     at a time, each held as two bf16 boxes (hi = bf16(x), lo = bf16(x - hi),
//     16 significant bits together).  To the MMA issuer such a chunk is a
//     64-key chunk whose keys 0-31 are the hi rows and 32-63 the lo rows: the
//     softmax adds the two halves of S in fp32 (s q·k̄ = S_hi + S_lo) and writes
//     the same P for both halves, so P V adds P v̄_hi + P v̄_lo.  The
//     compensated logits and values thus keep the fp32 centroids to about
//     2^-17 relative.  The per-column bias is log2|b| (weight |b|), -inf for
//     clusters that are exact for a or empty.  Exact and centroid boxes never
//     share a chunk.
// Warp roles (12 warps):
//   warp 0      TMA producer: Q tiles once, then chunk boxes into a 4-stage
//               ring.  It publishes each stage's chunk descriptor (box count,
//               valid rows per box, centroid or not, bias) in shared memory
//               and ends the sequence with an empty descriptor.  With G
//               (gather) Q, K and V stay in their original token order: the
//               producer walks the box sequence two chunks ahead of the ring,
//               keeping each chunk's descriptor in a small shared-memory ring
//               and fetching the original index of each of its permuted rows
//               (k_perm) with 4-byte cp.async copies into a matching index
//               ring, so the index latency overlaps the chunks before it; at
//               issue the lanes check and convert the indices and the elected
//               lane fetches rows four at a time with TMA tile::gather4 into
//               the same swizzled layout (§3.1's permutation folded into the
//               loads; no permuted copies).
//   warp 1      MMA issuer (one elected lane of the warp): S_t = Q_t K^T into
//               one of two TMEM buffers per tile, then O_t += P_t V with P_t
//               read from TMEM.  Issue order
//               QK_A(0) QK_B(0) QK_A(1) QK_B(1) | PV_A(c) QK_A(c+2) PV_B(c) QK_B(c+2) | ...
//               so the next chunk's scores are ready while the softmax works.
//   warps 4-7   softmax of tile A, warps 8-11 softmax of tile B: one thread
//               per query row (= TMEM lane).  Online softmax in base 2 on the
//               raw scores: an exact chunk is read from TMEM once (max, then
//               exponent, from registers); the exponent argument is one packed
//               FMA per score pair; the running max only moves (and O is
//               rescaled in TMEM) when it grows by more than 2^8.
// TMEM (512 columns): S_A0 [0,64), S_A1 [64,128), S_B0 [128,192), S_B1 [192,256),
// O_A [256,384), O_B [384,512); P (bf16 pairs) overwrites the first half of its S buffer.
#include <mutex>

#include "ear_internal.cuh"
#include "sm100.cuh"

namespace ear {
namespace {

using namespace sm100;

constexpr int kTileRows = 128;
constexpr int kTiles = 2;
constexpr int kUnitRows = kTileRows * kTiles;
constexpr int kBox = 32;                 // rows per TMA box
constexpr int kBoxes = 2;                // boxes per chunk
constexpr int kChunk = kBox * kBoxes;    // keys per chunk
constexpr int kStages = 4;               // K/V ring depth (chunks)
constexpr int kLook = 2;                 // gather: chunks walked ahead of the issue
constexpr int kRing = 4;                 // gather: descriptor / index ring (> kLook)
constexpr int kSBufs = 2;                // S buffers per tile: Q K^T of chunk c+1 runs
                                         // while the softmax works on chunk c
constexpr int kThreads = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.0f;  // move the running max only when it grows by > 2^8
constexpr int kTableMax = 2048;   // block list / key offsets staged in shared memory up to this
// Register split (setmaxnreg): warps 0-3 (producer, MMA issuer, 2 idle) drop
// to regs_low<D>(), the two softmax warpgroups rise to kRegsHigh.  The sum stays
// within the 168 registers x 384 threads the kernel is launched with; the
// launcher checks the compiled count before every launch.
template <int D>
constexpr int regs_low() { return D == 128 ? 72 : 64; }
constexpr int kRegsHigh = 216;
constexpr int kRegsLaunch = 168;
static_assert(128 * regs_low<128>() + 256 * kRegsHigh <= kThreads * kRegsLaunch, "register split");
static_assert(128 * regs_low<64>() + 256 * kRegsHigh <= kThreads * kRegsLaunch, "register split");

// barrier slots
constexpr int kBarKvFull = 0;                     // + stage
constexpr int kBarKvEmpty = kStages;              // + stage
constexpr int kBarQFull = 2 * kStages;
constexpr int kBarSFull = kBarQFull + 1;          // + tile * kSBufs + buffer
constexpr int kBarPFull = kBarSFull + kTiles * kSBufs;  // + tile * kSBufs + buffer
// O_t += P V of chunk c done: one barrier per (tile, S buffer of c).  With two
// S buffers a softmax warp at chunk c only knows that P V of chunk c-2 has
// finished; per-buffer barriers keep every parity wait within one phase.
constexpr int kBarODone = kBarPFull + kTiles * kSBufs;  // + tile * kSBufs + buffer
constexpr int kBarDrain = kBarODone + kTiles * kSBufs;  // teardown: every MMA issued has finished
constexpr int kNumBars = kBarDrain + 1;

// Chunk descriptor published by the producer for each stage.
struct ChunkInfo {
  int32_t nbox;          // 0 = no more chunks
  int32_t comp;          // centroid chunk
  int32_t valid[kBoxes]; // valid rows of each box (1..32)
};

// Gather: a chunk walked ahead of its issue (the producer's own ring).
struct AheadDesc {
  int32_t nbox, comp, r0, r1, v0, v1, comp_first, pad;
};

template <int D>
struct Layout {
  static constexpr int kHalfBytes = kTileRows * 128;  // Q tile: 128 rows x 64 bf16 per half
  static constexpr int kTileBytes = kHalfBytes * (D / 64);
  static constexpr int kSHalf = kChunk * 128;         // K / V stage: 64 rows x 64 bf16 per half
  static constexpr int kStageBytes = kSHalf * (D / 64);
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTiles * kTileBytes;
  static constexpr int kV = kK + kStages * kStageBytes;
  static constexpr int kBias = kV + kStages * kStageBytes;      // [stage][kChunk] float
  static constexpr int kInfo = kBias + kStages * kChunk * 4;    // [stage] ChunkInfo
  static constexpr int kList = kInfo + kStages * 32;              // unit's exact key clusters
  static constexpr int kKoff = kList + kTableMax * 4;             // slice's key offsets
  static constexpr int kExact = kKoff + kTableMax * 4;            // unit's row of the mask
  static constexpr int kQIdx = kExact + kTableMax;                // gather: Q row coordinates
  static constexpr int kGIdx = kQIdx + kUnitRows * 4;             // gather: kRing chunks' K / V rows
  static constexpr int kAhead = kGIdx + kRing * kChunk * 4;       // gather: kRing AheadDesc
  static constexpr int kBar = kAhead + kRing * (int)sizeof(AheadDesc);
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16 + 1024;  // + slack to align the base to 1024
};

struct TcParams {
  const int32_t* q_off;
  const int32_t* k_off;
  const int32_t* q_perm;
  const int32_t* k_perm;  // gather: original index of each permuted key
  const uint8_t* exact;
  const int32_t* blk_off;
  const int32_t* blk_list;
  const int2* items;
  const int32_t* count;
  int64_t max_items;
  int64_t Nq, Nk;
  int Cq, Ck, Ck_pad;
  float qk_scale;  // scale * log2(e)
  int compensate;
  uint16_t* O;
  float* lse;
  int* status;
};

// Box sequence of one unit (producer only): the rows of each exact key
// cluster in 32-row boxes, then the centroids in 32-row boxes.
struct Boxes {
  const int32_t* list;
  const int32_t* koff;
  int32_t e, e1, pos, end;
  int32_t comp_next, Ck, Nk;
  int compensate;
  int* status;

  // list: the unit's exact key clusters [0, n); koff: the slice's key offsets.
  __device__ void init(const TcParams& p, const int32_t* list_, int n, const int32_t* koff_) {
    list = list_;
    koff = koff_;
    e = 0;
    e1 = n;
    pos = end = 0;
    comp_next = 0;
    Ck = p.Ck;
    Nk = (int32_t)p.Nk;
    compensate = p.compensate;
    status = p.status;
  }
  // Next box: first row (key row in the slice, or centroid index), valid
  // rows, and whether it is a centroid box.  False when none is left.
  __device__ bool next(int32_t& row, int& valid, bool& comp) {
    while (pos >= end && e < e1) {
      const int b = list[e++];
      if (b < 0 || b >= Ck) {
        latch(status, EAR_ERR_DEVICE);
        continue;
      }
      pos = koff[b];
      end = koff[b + 1];
      if (pos < 0 || end > Nk || end < pos) {
        latch(status, EAR_ERR_DEVICE);
        pos = end = 0;
      }
    }
    if (pos < end) {
      row = pos;
      valid = min(kBox, end - pos);
      pos += valid;
      comp = false;
      return true;
    }
    if (compensate && comp_next < Ck) {
      row = comp_next;  // centroid index; its hi / lo boxes sit at rows 2 row, 2 row + 32
      valid = min(kBox, Ck - comp_next);
      comp_next += kBox;
      comp = true;
      return true;
    }
    return false;
  }
};

__device__ __forceinline__ unsigned long long pack2(uint32_t lo, uint32_t hi) {
  return (unsigned long long)lo | ((unsigned long long)hi << 32);
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float lo_f(unsigned long long x) { return __uint_as_float((uint32_t)x); }
__device__ __forceinline__ float hi_f(unsigned long long x) {
  return __uint_as_float((uint32_t)(x >> 32));
}

// max of 32 raw scores, columns >= valid excluded
__device__ __forceinline__ float box_max_raw(const uint32_t (&v)[32], int valid) {
  float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  if (valid >= 32) {
#pragma unroll
    for (int j = 0; j < 32; ++j) m[j & 3] = fmaxf(m[j & 3], __uint_as_float(v[j]));
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      m[j & 3] = fmaxf(m[j & 3], j < valid ? __uint_as_float(v[j]) : -INFINITY);
  }
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// max of 32 scaled-and-biased scores (centroid box)
__device__ __forceinline__ float box_max_bias(const uint32_t (&v)[32], const float* bias,
                                              float scale, int valid) {
  float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float z = fmaf(__uint_as_float(v[j]), scale, bias[j]);
    m[j & 3] = fmaxf(m[j & 3], j < valid ? z : -INFINITY);
  }
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// p = 2^(score * scale + bias_j - m) for 32 columns (bias from shared memory,
// neg = -m), packed to bf16 pairs; returns the two partial row sums as a pair.
__device__ __forceinline__ unsigned long long box_exp(const uint32_t (&v)[32], const float* bias,
                                                      float neg, unsigned long long scale2,
                                                      int valid, uint32_t (&pk)[16]) {
  unsigned long long sum = 0;
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const float2 b2 = *reinterpret_cast<const float2*>(bias + j);
    const unsigned long long sh = pack2(__float_as_uint(b2.x + neg), __float_as_uint(b2.y + neg));
    const unsigned long long z = fma2(pack2(v[j], v[j + 1]), scale2, sh);
    float p0 = ex2(lo_f(z)), p1 = ex2(hi_f(z));
    if (valid < 32) {
      p0 = j < valid ? p0 : 0.f;
      p1 = j + 1 < valid ? p1 : 0.f;
    }
    sum = add2(sum, pack2(__float_as_uint(p0), __float_as_uint(p1)));
    pk[j / 2] = pack_bf16x2(p0, p1);
  }
  return sum;
}

// box_exp with one shift pair for every column (exact box)
__device__ __forceinline__ unsigned long long box_exp_c(const uint32_t (&v)[32],
                                                        unsigned long long sh,
                                                        unsigned long long scale2, int valid,
                                                        uint32_t (&pk)[16]) {
  unsigned long long sum0 = 0, sum1 = 0;
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const unsigned long long z = fma2(pack2(v[j], v[j + 1]), scale2, sh);
    float p0 = ex2(lo_f(z)), p1 = ex2(hi_f(z));
    if (valid < 32) {
      p0 = j < valid ? p0 : 0.f;
      p1 = j + 1 < valid ? p1 : 0.f;
    }
    const unsigned long long pr = pack2(__float_as_uint(p0), __float_as_uint(p1));
    if (j & 2) sum1 = add2(sum1, pr); else sum0 = add2(sum0, pr);
    pk[j / 2] = pack_bf16x2(p0, p1);
  }
  return add2(sum0, sum1);
}

template <int D, bool G>
__device__ __forceinline__ void producer_role(
    const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
    const CUtensorMap& tmKc, const CUtensorMap& tmVc, const TcParams& p, uint8_t* smem, int64_t h,
    int a, int32_t row0, int ntiles, int qrows, int lane, volatile int* abort) {
  using L = Layout<D>;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  float* bias = reinterpret_cast<float*>(smem + L::kBias);
  ChunkInfo* info = reinterpret_cast<ChunkInfo*>(smem + L::kInfo);
  {
    {
    const uint8_t* exact_row = p.exact + (h * p.Cq + a) * (int64_t)p.Ck;
    const int32_t* koff = p.k_off + h * (int64_t)(p.Ck + 1);
    const bool leader = elect_one();  // issues the TMA copies (operands stay warp-uniform)
    int32_t* qidx = reinterpret_cast<int32_t*>(smem + L::kQIdx);
    if (G) {  // the unit's query rows; rows past the unit repeat its last row
      for (int r = lane; r < ntiles * kTileRows; r += 32)
        qidx[r] = gather_row(p.q_perm, h * p.Nq + row0 + min(r, qrows - 1), h, p.Nq, p.status);
      __syncwarp();
    }
    if (leader) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bars[kBarQFull], ntiles * L::kTileBytes);
      for (int t = 0; t < ntiles; ++t) {
        uint8_t* qdst = smem + L::kQ + t * L::kTileBytes;
        if (G) {
          for (int g = 0; g < kTileRows / 4; ++g) {
            const int4 rr = *reinterpret_cast<const int4*>(qidx + t * kTileRows + 4 * g);
            for (int hf = 0; hf < D / 64; ++hf)
              tma_gather4(qdst + hf * L::kHalfBytes + g * 4 * 128, &tmQ, &bars[kBarQFull],
                          64 * hf, rr);
          }
        } else {
          for (int hf = 0; hf < D / 64; ++hf)
            tma_load_2d(qdst + hf * L::kHalfBytes, &tmQ, &bars[kBarQFull], 64 * hf,
                        (int32_t)(h * p.Nq) + row0 + kTileRows * t);
        }
      }
    }
    // Stage the unit's block list and the slice's key offsets in shared memory
    // (the box walk below would otherwise chase them through L2 per block).
    const int32_t* bo = p.blk_off + h * (int64_t)(p.Cq + 1);
    const int32_t e0 = bo[a], nlist = bo[a + 1] - bo[a];
    const int32_t* glist = p.blk_list + h * (int64_t)p.Cq * p.Ck + e0;
    const int32_t* list = glist;
    const int32_t* koff_t = koff;
    const uint8_t* exact_t = exact_row;
    if (nlist <= kTableMax && p.Ck + 1 <= kTableMax && nlist >= 0) {
      int32_t* sl = reinterpret_cast<int32_t*>(smem + L::kList);
      int32_t* sk = reinterpret_cast<int32_t*>(smem + L::kKoff);
      uint8_t* se = smem + L::kExact;
      for (int i = lane; i < nlist; i += 32) sl[i] = glist[i];
      for (int i = lane; i <= p.Ck; i += 32) sk[i] = koff[i];
      for (int i = lane; i < p.Ck; i += 32) se[i] = exact_row[i];
      __syncwarp();
      list = sl;
      koff_t = sk;
      exact_t = se;
    }
    Boxes it;
    it.init(p, list, max(nlist, 0), koff_t);
    int32_t brow = 0;
    int bval = 0;
    bool bcomp = false;
    bool have = it.next(brow, bval, bcomp);  // the box that opens the next chunk
    // The next chunk: up to four boxes of the same kind, held in registers
    // (static indices).  It is gathered while the ring slot is still busy.
    int comp = 0, nbox = 0;
    int32_t r0 = 0, r1 = 0, comp_first = 0;
    int v0 = 0, v1 = 0;
    auto gather = [&]() {
      comp = have && bcomp ? 1 : 0;
      nbox = 0;
      r0 = r1 = 0;
      v0 = v1 = 0;
      comp_first = brow;
#pragma unroll
      for (int k = 0; k < kBoxes; ++k) {
        if (!(have && (bcomp ? 1 : 0) == comp)) break;
        if (k > 0 && comp) break;  // a centroid chunk is one group of 32 (hi + lo boxes)
        if (k == 0) { r0 = brow; v0 = bval; }
        if (k == 1) { r1 = brow; v1 = bval; }
        nbox = k + 1;
        have = it.next(brow, bval, bcomp);
      }
    };
    // G: chunk j walked ahead -> descriptor ring slot j % kRing, and its rows'
    // k_perm entries copied asynchronously into the index ring (rows past a
    // box's valid count repeat its last row); one commit group per chunk
    AheadDesc* ahead = reinterpret_cast<AheadDesc*>(smem + L::kAhead);
    int32_t* gring = reinterpret_cast<int32_t*>(smem + L::kGIdx);
    auto walk_ahead = [&](int j) {
      gather();
      const int slot = j % kRing;
      if (lane == 0) ahead[slot] = AheadDesc{nbox, comp, r0, r1, v0, v1, comp_first, 0};
      if (!comp) {
        const int32_t* kp = p.k_perm + h * p.Nk;
        if (nbox > 0) cp_async4(gring + slot * kChunk + lane, kp + r0 + min(lane, v0 - 1));
        if (nbox > 1) cp_async4(gring + slot * kChunk + 32 + lane, kp + r1 + min(lane, v1 - 1));
      }
      cp_async_commit();
    };
    if (G) {
      for (int j = 0; j < kLook; ++j) walk_ahead(j);
    } else {
      gather();
    }
    int issued = 0;
    for (int c = 0;; ++c) {
      const int s = c % kStages;
      if (c >= kStages && !mbar_wait(&bars[kBarKvEmpty + s], ((c / kStages) - 1) & 1, abort))
        break;
      issued = c + 1;
      if (G) {  // this chunk's descriptor, walked kLook chunks ago
        __syncwarp();
        const AheadDesc d = ahead[c % kRing];
        nbox = d.nbox;
        comp = d.comp;
        r0 = d.r0;
        r1 = d.r1;
        v0 = d.v0;
        v1 = d.v1;
        comp_first = d.comp_first;
      }
      if (comp) {  // bias of the chunk's columns (centroids comp_first ...)
        for (int j = lane; j < kChunk; j += 32) {
          float bv = -INFINITY;
          const int bx = j / kBox;
          const int vb = bx == 0 ? v0 : v1;
          if (bx < nbox && (j % kBox) < vb) {
            const int b = comp_first + j;
            const int32_t cnt = koff_t[b + 1] - koff_t[b];
            if (!exact_t[b] && cnt > 0) bv = __log2f((float)cnt);
          }
          bias[s * kChunk + j] = bv;
        }
      }
      __syncwarp();
      if (leader) {
        ChunkInfo* ci = &info[s];
        ci->nbox = nbox;
        ci->comp = comp;
        ci->valid[0] = v0;
        ci->valid[1] = v1;
        if (nbox == 0)
          mbar_arrive(&bars[kBarKvFull + s]);  // end of the sequence
        else
          mbar_arrive_expect_tx(&bars[kBarKvFull + s], 2 * (comp ? 2 : nbox) * kBox * D * 2);
      }
      if (G && !comp) {
        // this lane's index copies of chunk c have landed (kLook - 1 later chunks may not);
        // each lane checks its two entries and turns them into row coordinates
        cp_async_wait<kLook - 1>();
        int32_t* gidx = gring + (c % kRing) * kChunk;
        for (int k = 0; k < nbox; ++k) {
          int32_t o = gidx[lane + 32 * k];
          if (o < 0 || o >= p.Nk) {
            latch(p.status, EAR_ERR_DEVICE);
            o = 0;
          }
          gidx[lane + 32 * k] = (int32_t)(h * p.Nk) + o;
        }
        __syncwarp();
        uint8_t* kdst = smem + L::kK + s * L::kStageBytes;
        uint8_t* vdst = smem + L::kV + s * L::kStageBytes;
        if (leader) {
          for (int g = 0; g < nbox * (kBox / 4); ++g) {
            const int4 rr = *reinterpret_cast<const int4*>(gidx + 4 * g);
#pragma unroll
            for (int hf = 0; hf < D / 64; ++hf) {
              tma_gather4(kdst + hf * L::kSHalf + g * 4 * 128, &tmK, &bars[kBarKvFull + s],
                          64 * hf, rr);
              tma_gather4(vdst + hf * L::kSHalf + g * 4 * 128, &tmV, &bars[kBarKvFull + s],
                          64 * hf, rr);
            }
          }
        }
      } else {
        const CUtensorMap* mk = comp ? &tmKc : &tmK;
        const CUtensorMap* mv = comp ? &tmVc : &tmV;
        const int32_t base = comp ? (int32_t)(h * p.Ck_pad) : (int32_t)(h * p.Nk);
        const int nphys = comp ? 2 : nbox;  // a centroid chunk loads its hi and lo boxes
        uint8_t* kdst = smem + L::kK + s * L::kStageBytes;
        uint8_t* vdst = smem + L::kV + s * L::kStageBytes;
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx) {
          const int32_t rw = comp ? 2 * r0 + bx * kBox : (bx == 0 ? r0 : r1);
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf) {
            if (bx < nphys && leader) {
              tma_load_2d(kdst + hf * L::kSHalf + bx * kBox * 128, mk, &bars[kBarKvFull + s],
                          64 * hf, base + rw);
              tma_load_2d(vdst + hf * L::kSHalf + bx * kBox * 128, mv, &bars[kBarKvFull + s],
                          64 * hf, base + rw);
            }
          }
        }
      }
      __syncwarp();
      if (nbox == 0) break;
      if (G)
        walk_ahead(c + kLook);
      else
        gather();
    }
    if (G) cp_async_wait_all();  // no index copy outlives the producer
    if (*abort) {  // let issued loads land before the CTA exits
      mbar_wait_drain(&bars[kBarQFull], 0);
      for (int c = issued - 1; c >= 0 && c >= issued - kStages; --c)
        mbar_wait_drain(&bars[kBarKvFull + c % kStages], (c / kStages) & 1);
    }
    }
  }
}

template <int D>
__device__ __forceinline__ void mma_role(const TcParams& p, uint8_t* smem, uint32_t tmem, int ntiles,
                                         volatile int* abort) {
  using L = Layout<D>;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  ChunkInfo* info = reinterpret_cast<ChunkInfo*>(smem + L::kInfo);
  {
    {
      // One elected lane runs the whole loop: waits, MMAs and commits.  (A
      // warp-wide loop with a per-MMA lane predicate was measurably slower.)
      const uint32_t idesc_pv = idesc_bf16(128, D, true);
      if (elect_one()) {
        // S of tile t, buffer b: TMEM columns [128 t + 64 b, +64); O_t: [256 + 128 t, +128)
        // n = keys of the chunk (32 or 64; a centroid chunk is 64: hi rows, then lo rows)
        auto issue_qk = [&](int t, int buf, int s, int n) {
          const uint32_t idesc = idesc_bf16(128, (uint32_t)n, false);
          const uint64_t qd = desc_sw128(smem_u32(smem + L::kQ + t * L::kTileBytes), 16, 1024);
          const uint64_t kd = desc_sw128(smem_u32(smem + L::kK + s * L::kStageBytes), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qo = ((kk / 4) * L::kHalfBytes + (kk % 4) * 32) >> 4;
            const uint32_t ko = ((kk / 4) * L::kSHalf + (kk % 4) * 32) >> 4;
            mma_ss(tmem + kTileRows * t + kChunk * buf, qd + qo, kd + ko, idesc, kk > 0 ? 1u : 0u);
          }
        };
        auto issue_pv = [&](int t, int buf, int s, int n, bool first) {
          const uint64_t vd = desc_sw128(smem_u32(smem + L::kV + s * L::kStageBytes), L::kSHalf, 1024);
          const int nk = n / 16;
#pragma unroll
          for (int kk = 0; kk < kChunk / 16; ++kk) {
            if (kk < nk)
              mma_ts(tmem + 256 + kTileRows * t, tmem + kTileRows * t + kChunk * buf + kk * 8,
                     vd + ((kk * 2048) >> 4), idesc_pv, (first && kk == 0) ? 0u : 1u);
          }
        };
        bool ok = mbar_wait(&bars[kBarQFull], 0, abort) && mbar_wait(&bars[kBarKvFull], 0, abort);
        auto keys_of = [&](int st) { return (info[st].comp ? 2 : info[st].nbox) * kBox; };
        // n0, n1: keys of chunks c and c+1 (0 = past the end)
        int n0 = ok ? keys_of(0) : 0, n1 = 0;
        if (ok && n0 > 0) {
          tc_fence_after();
          for (int t = 0; t < ntiles; ++t) {
            issue_qk(t, 0, 0, n0);
            mma_commit(&bars[kBarSFull + t * kSBufs]);
          }
          ok = mbar_wait(&bars[kBarKvFull + 1], 0, abort);
          n1 = ok ? keys_of(1) : 0;
          if (ok && n1 > 0) {
            tc_fence_after();
            for (int t = 0; t < ntiles; ++t) {
              issue_qk(t, 1, 1, n1);
              mma_commit(&bars[kBarSFull + t * kSBufs + 1]);
            }
          }
        }
        for (int c = 0; ok && n0 > 0; ++c) {
          const int s = c % kStages, buf = c & 1;
          const int s2 = (c + 2) % kStages;
          int n2 = 0;
          for (int t = 0; t < ntiles && ok; ++t) {
            ok = mbar_wait(&bars[kBarPFull + t * kSBufs + buf], (c >> 1) & 1, abort);
            if (!ok) break;
            tc_fence_after();
            issue_pv(t, buf, s, n0, c == 0);
            mma_commit(&bars[kBarODone + t * kSBufs + buf]);
            if (t == ntiles - 1) mma_commit(&bars[kBarKvEmpty + s]);
            if (t == 0 && n1 > 0) {
              ok = mbar_wait(&bars[kBarKvFull + s2], ((c + 2) / kStages) & 1, abort);
              if (!ok) break;
              n2 = keys_of(s2);
              tc_fence_after();
            }
            if (n2 > 0) {  // chunk c+2 into the buffer P V of chunk c has just read
              issue_qk(t, buf, s2, n2);
              mma_commit(&bars[kBarSFull + t * kSBufs + buf]);
            }
          }
          n0 = n1;
          n1 = n2;
        }
        // every MMA issued above has finished before TMEM is released
        mma_commit(&bars[kBarDrain]);
      }
      __syncwarp();
      mbar_wait_drain(&bars[kBarDrain], 0);
    }
  }
}

template <int D>
__device__ __forceinline__ void softmax_role(const TcParams& p, uint8_t* smem, uint32_t tmem,
                                             int64_t h, int32_t row0, int rows_a, int rows_b,
                                             int ntiles, int warp, int lane, volatile int* abort) {
  using L = Layout<D>;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  float* bias = reinterpret_cast<float*>(smem + L::kBias);
  ChunkInfo* info = reinterpret_cast<ChunkInfo*>(smem + L::kInfo);
  {
    const int t = (warp - 4) / 4;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // row within the tile = TMEM lane
    const int rows_t = t == 0 ? rows_a : rows_b;
    if (t < ntiles) {
      const uint32_t lane_bits = (uint32_t)(wq * 32) << 16;
      const uint32_t tS0 = tmem + lane_bits + kTileRows * t;  // S buffer 0 of this tile
      const uint32_t tO = tmem + lane_bits + 256 + kTileRows * t;
      const float scale = p.qk_scale;
      const unsigned long long scale2 = pack2(__float_as_uint(scale), __float_as_uint(scale));
      float m = -INFINITY;                  // running max (scaled, base 2)
      unsigned long long lsum = 0;          // running sum as two partial sums
      int c = 0;
      bool ok = true;
      for (;; ++c) {
        const int s = c % kStages;
        ok = mbar_wait_warp(&bars[kBarKvFull + s], (c / kStages) & 1, abort);
        if (!ok) break;
        const ChunkInfo* ci = &info[s];  // read in place (runtime box index)
        const int nbox = ci->nbox;
        const bool comp = ci->comp != 0;
        if (nbox == 0) break;
        const int buf = c & 1;
        const uint32_t tS = tS0 + kChunk * buf;
        ok = mbar_wait_warp(&bars[kBarSFull + t * kSBufs + buf], (c >> 1) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        const float* bs = bias + s * kChunk;
        bool resc = false;
        float corr = 1.f, m_use = m;
        if (!comp) {
          // exact chunk: one TMEM trip for both boxes (an unused box has
          // valid = 0), max and exponent from registers
          const int v0 = ci->valid[0], v1 = ci->valid[1];
          uint32_t x0[32], x1[32];
          tmem_ld32(tS, x0);
          tmem_ld32(tS + 32, x1);
          tmem_ld_wait();
          const float mx = fmaxf(box_max_raw(x0, v0), box_max_raw(x1, v1)) * scale;
          if (mx > m + kRescale || (m == -INFINITY && mx > -INFINITY)) {
            if (m != -INFINITY) {
              resc = true;
              corr = ex2(m - mx);
            }
            m_use = mx;
          }
          if (resc) lsum = pack2(__float_as_uint(lo_f(lsum) * corr), __float_as_uint(hi_f(lsum) * corr));
          const float neg = m_use == -INFINITY ? 0.f : -m_use;
          const unsigned long long n2 = pack2(__float_as_uint(neg), __float_as_uint(neg));
          const bool none = m_use == -INFINITY;  // every score -inf: p = 0
          uint32_t pk[16];
          lsum = add2(lsum, box_exp_c(x0, n2, scale2, none ? 0 : v0, pk));
          tmem_st16(tS, pk);
          if (nbox > 1) {
            lsum = add2(lsum, box_exp_c(x1, n2, scale2, none ? 0 : v1, pk));
            tmem_st16(tS + 16, pk);
          }
        } else {
          // centroid chunk: S columns 0-31 = Q k̄_hi^T, 32-63 = Q k̄_lo^T for 32
          // centroids; s q·k̄ = S_hi + S_lo in fp32, weight |b| through the bias
          const int v0 = ci->valid[0];
          uint32_t x0[32], x1[32];
          tmem_ld32(tS, x0);
          tmem_ld32(tS + 32, x1);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            x0[j] = __float_as_uint(__uint_as_float(x0[j]) + __uint_as_float(x1[j]));
          const float mx = box_max_bias(x0, bs, scale, v0);
          if (mx > m + kRescale || (m == -INFINITY && mx > -INFINITY)) {
            if (m != -INFINITY) {
              resc = true;
              corr = ex2(m - mx);
            }
            m_use = mx;
          }
          if (resc) lsum = pack2(__float_as_uint(lo_f(lsum) * corr), __float_as_uint(hi_f(lsum) * corr));
          const float neg = m_use == -INFINITY ? 0.f : -m_use;  // all scores -inf: p = 0 below
          uint32_t pk[16];
          lsum = add2(lsum, box_exp(x0, bs, neg, scale2, m_use == -INFINITY ? 0 : v0, pk));
          tmem_st16(tS, pk);       // P for the hi rows
          tmem_st16(tS + 16, pk);  // the same P for the lo rows
        }
        tmem_st_wait();
        if (__any_sync(0xffffffffu, resc)) {
          // P V of chunk c-1 (c-2 and earlier are done: S of chunk c was written after them)
          ok = mbar_wait_warp(&bars[kBarODone + t * kSBufs + ((c - 1) & 1)], ((c - 1) >> 1) & 1,
                              abort);
          if (!ok) break;
          tc_fence_after();
          for (int g = 0; g < D / 32; ++g) {
            uint32_t v[32];
            tmem_ld32(tO + 32 * g, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * corr);
            tmem_st32(tO + 32 * g, v);
          }
          tmem_st_wait();
        }
        m = m_use;
        tc_fence_before();
        mbar_arrive(&bars[kBarPFull + t * kSBufs + buf]);
      }
      // epilogue: O / l written at the queries' original positions
      const float l = lo_f(lsum) + hi_f(lsum);
      const int32_t prow = row0 + kTileRows * t + r;
      const int32_t orig = r < rows_t ? p.q_perm[h * p.Nq + prow] : -1;
      const bool valid = orig >= 0 && orig < p.Nq;
      if (r < rows_t && !valid) latch(p.status, EAR_ERR_DEVICE);
      // the last two chunks' P V (either may still run: nothing later waited on them)
      bool have_o = ok && c > 0 &&
                    mbar_wait_warp(&bars[kBarODone + t * kSBufs + ((c - 1) & 1)], ((c - 1) >> 1) & 1,
                                   abort);
      if (have_o && c > 1)
        have_o = mbar_wait_warp(&bars[kBarODone + t * kSBufs + ((c - 2) & 1)], ((c - 2) >> 1) & 1,
                                abort);
      if (have_o) tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint16_t* orow = p.O + ((int64_t)h * p.Nq + (valid ? orig : 0)) * D;
      for (int g = 0; g < D / 32; ++g) {
        uint32_t v[32];
        if (have_o) {
          tmem_ld32(tO + 32 * g, v);
          tmem_ld_wait();
        }
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2)
            pk[j / 2] = have_o ? pack_bf16x2(__uint_as_float(v[j]) * inv,
                                             __uint_as_float(v[j + 1]) * inv)
                               : 0u;
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * g);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            dst[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
      }
      if (valid && p.lse != nullptr)
        p.lse[h * p.Nq + orig] = (have_o && l > 0.f) ? (m + __log2f(l)) * kLn2 : -INFINITY;
    }
  }

}

template <int D, bool G>
__global__ void __launch_bounds__(kThreads, 1)
at_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKc,
      const __grid_constant__ CUtensorMap tmVc, const TcParams p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int64_t h = blockIdx.y;
  const int64_t slot = blockIdx.x;
  if (slot >= p.count[h]) return;
  const int2 item = p.items[h * p.max_items + slot];
  const int a = item.x;
  const int32_t row0 = item.y;
  const int32_t qend = p.q_off[h * (int64_t)(p.Cq + 1) + a + 1];
  if (row0 < 0 || qend > p.Nq || row0 >= qend) {
    if (threadIdx.x == 0) latch(p.status, EAR_ERR_DEVICE);
    return;
  }
  const int rows_a = min(kTileRows, qend - row0);
  const int rows_b = max(0, min(kTileRows, qend - row0 - kTileRows));
  const int ntiles = rows_b > 0 ? 2 : 1;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  float* bias = reinterpret_cast<float*>(smem + L::kBias);
  ChunkInfo* info = reinterpret_cast<ChunkInfo*>(smem + L::kInfo);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[kBarKvFull + s], 1);
      mbar_init(&bars[kBarKvEmpty + s], 1);
    }
    mbar_init(&bars[kBarQFull], 1);
    mbar_init(&bars[kBarDrain], 1);
    for (int t = 0; t < kTiles; ++t) {
      for (int b = 0; b < kSBufs; ++b) {
        mbar_init(&bars[kBarSFull + t * kSBufs + b], 1);
        mbar_init(&bars[kBarPFull + t * kSBufs + b], kTileRows);
        mbar_init(&bars[kBarODone + t * kSBufs + b], 1);
      }
    }
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Each role ends with its own teardown (a CTA-wide bar.sync, then warp 0
  // frees TMEM), so no code runs under both register budgets.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(regs_low<D>()));
    if (warp == 0) {
      producer_role<D, G>(tmQ, tmK, tmV, tmKc, tmVc, p, smem, h, a, row0, ntiles,
                          rows_a + rows_b, lane, abort);
    } else if (warp == 1) {
      mma_role<D>(p, smem, tmem, ntiles, abort);
    }
    tc_fence_before();
    asm volatile("bar.sync 0;" ::: "memory");
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
      if (lane == 0 && *abort) latch(p.status, EAR_ERR_TIMEOUT);
    }
    return;
  }
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsHigh));
  softmax_role<D>(p, smem, tmem, h, row0, rows_a, rows_b, ntiles, warp, lane, abort);
  tc_fence_before();
  asm volatile("bar.sync 0;" ::: "memory");
}

// Key / value centroids as bf16 pairs: per slice, groups of 32 centroids, each
// group 32 rows of hi = bf16(x) followed by 32 rows of lo = bf16(x - hi)
// (x - hi is exact in fp32); rows past C_k are zero.  rows = 64 per group.
__global__ void at_centroids_bf16(const float* __restrict__ kc, const float* __restrict__ vc,
                                  uint16_t* __restrict__ kc16, uint16_t* __restrict__ vc16,
                                  int Ck, int rows, int D, int64_t total) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const int64_t hr = e / D;
  const int k = (int)(e % D);
  const int64_t h = hr / rows;
  const int r = (int)(hr % rows);
  const int c = (r / 64) * 32 + (r % 32);
  const bool lo = (r % 64) >= 32;
  uint16_t ko = 0, vo = 0;
  if (c < Ck) {
    const float kx = kc[(h * Ck + c) * D + k], vx = vc[(h * Ck + c) * D + k];
    const uint16_t kh = f32_to_bf16(kx), vh = f32_to_bf16(vx);
    ko = lo ? f32_to_bf16(kx - bf16_to_f32(kh)) : kh;
    vo = lo ? f32_to_bf16(vx - bf16_to_f32(vh)) : vh;
  }
  kc16[e] = ko;
  vc16[e] = vo;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D bf16 map over [rows][d], 64-column x box_rows boxes, 128-byte swizzle,
// zero fill past the last row.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool G>
ear_status tc_t(const AttnArgs& a, int2* items, int32_t* count, int64_t max_items,
                uint16_t* kc16, uint16_t* vc16, int ck_pad, cudaStream_t s) {
  using L = Layout<D>;
  const int64_t total = a.bh * (int64_t)ck_pad * D;
  at_centroids_bf16<<<(unsigned)ceil_div(total, 256), 256, 0, s>>>(a.k_cent, a.v_cent, kc16, vc16,
                                                                   a.c_k, ck_pad, D, total);
  EAR_TRY(after_launch());
  CUtensorMap mq, mk, mv, mkc, mvc;
  // gather: one-row boxes (tile::gather4 fetches four of them per copy)
  if (!make_map(&mq, a.Q, a.bh * a.n_q, D, G ? 1 : kTileRows) ||
      !make_map(&mk, a.K, a.bh * a.n_k, D, G ? 1 : kBox) ||
      !make_map(&mv, a.V, a.bh * a.n_k, D, G ? 1 : kBox) ||
      !make_map(&mkc, kc16, a.bh * ck_pad, D, kBox) ||
      !make_map(&mvc, vc16, a.bh * ck_pad, D, kBox))
    return EAR_ERR_CUDA;
  TcParams p;
  p.q_off = a.q_off;
  p.k_off = a.k_off;
  p.q_perm = a.q_perm;
  p.k_perm = a.k_perm;
  p.exact = a.exact;
  p.blk_off = a.blk_off;
  p.blk_list = a.blk_list;
  p.items = items;
  p.count = count;
  p.max_items = max_items;
  p.Nq = a.n_q;
  p.Nk = a.n_k;
  p.Cq = a.c_q;
  p.Ck = a.c_k;
  p.Ck_pad = ck_pad;
  p.qk_scale = a.scale * kLog2e;
  p.compensate = a.flags & EAR_COMPENSATE;
  p.O = static_cast<uint16_t*>(a.O);
  p.lse = a.lse;
  p.status = device_status_word();
  EAR_CUDA(cudaFuncSetAttribute(at_tc<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                L::kBytes));
  // setmaxnreg.inc waits until the block's launch registers cover the split:
  // refuse to launch a build whose allocation does not.
  cudaFuncAttributes fa;
  EAR_CUDA(cudaFuncGetAttributes(&fa, at_tc<D, G>));
  if (fa.numRegs * kThreads < 128 * regs_low<D>() + 256 * kRegsHigh) return EAR_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)max_items, (unsigned)a.bh);
  at_tc<D, G><<<grid, kThreads, L::kBytes, s>>>(mq, mk, mv, mkc, mvc, p);
  return after_launch();
}

}  // namespace

// Rows of the bf16 centroid buffer per slice: 64 (32 hi + 32 lo) per group of 32.
int64_t attention_tc_ck_pad(int32_t c_k) { return ceil_div(c_k, kBox) * 2 * kBox; }

int64_t attention_tc_items_per_slice(int64_t n_q, int32_t c_q) {
  return ceil_div(n_q, kUnitRows) + c_q;
}

ear_status attention_tc_run(const AttnArgs& a, int2* items, int32_t* count, int64_t max_items,
                            uint16_t* kc16, uint16_t* vc16, cudaStream_t s) {
  const int ck_pad = (int)attention_tc_ck_pad(a.c_k);
  // TMA row coordinates are int32
  if (a.bh * a.n_q > INT32_MAX || a.bh * a.n_k > INT32_MAX || a.bh * ck_pad > INT32_MAX)
    return EAR_ERR_UNSUPPORTED;
  EAR_TRY(attention_plan(a.q_off, a.bh, a.c_q, kUnitRows, max_items, items, count, s));
  if (a.k_perm != nullptr)
    return a.d == 64 ? tc_t<64, true>(a, items, count, max_items, kc16, vc16, ck_pad, s)
                     : tc_t<128, true>(a, items, count, max_items, kc16, vc16, ck_pad, s);
  return a.d == 64 ? tc_t<64, false>(a, items, count, max_items, kc16, vc16, ck_pad, s)
                   : tc_t<128, false>(a, items, count, max_items, kc16, vc16, ck_pad, s);
}

}  // namespace ear
