// moe_mega.cuh -- the whole block as one persistent launch, for few tokens
// (B <= 8: one 8-column token tile in every phase).
//
// The four phases of the multi-kernel path -- dense front (router, latent,
// shared gate/up, plus the routing CTA), expert gate/up, expert down, latent
// tail -- become one ordered list of pieces behind one cursor.  Every CTA's
// producer walks that list: it streams each piece's weight tiles as soon as
// it holds the piece, and issues the piece's activation copies once the phase
// it depends on is complete, which it learns from completion counters that
// the finalising CTAs raise with release semantics:
//
//   expert gate/up  needs the routing (flag) and every latent row block (z)
//   expert down     needs every expert gate/up matrix (h)
//   latent tail     needs every expert down matrix (y) and every shared row
//                   block (h_s)
//
// So there are no kernel boundaries: a CTA that finishes its front pieces
// starts streaming expert tiles while others still finish theirs, and only the
// consumers wait on the counters.  A piece only waits on pieces earlier in the
// list, all held by running CTAs whose consumers need nothing from their own
// producer to finish them; and a consumer settles its split-K ticket before
// the phase changes, so no finalisation a later phase waits for is left
// pending behind that wait.  Every wait is bounded.
#pragma once
#include "moe_engine.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// producer

struct MegaProd {
  int stage;
  uint32_t ephase;
  bool dep_ok[KIND_COUNT];
  bool routed;
  int V;  // virtual experts (token groups of routed experts)
  Space sp[KIND_COUNT];
  int base[KIND_COUNT + 1];  // first list index of each phase; base[4] = list length
  int grabbed;               // lane 0: result of the grab in flight
  bool in_flight;
};

// Blocking: phase KIND's activations may be read.
template <int KIND>
__device__ __forceinline__ void mega_wait_deps(const MegaParams& mp, const MegaProd& st, int lane) {
  const Params& pf = mp.k[KIND_FRONT];
  if (KIND == KIND_FRONT) {
    pdl_wait();  // the previous forward is over
    pdl_trigger();
  } else if (KIND == KIND_EGU) {
    wait_count(pf.done + 0, pf.RB_lat, pf.err, lane);
  } else if (KIND == KIND_EDN) {
    wait_count(pf.done + 2, st.V * mp.k[KIND_EGU].RB, pf.err, lane);
  } else {
    wait_count(pf.done + 3, st.V * mp.k[KIND_EDN].RB, pf.err, lane);
    wait_count(pf.done + 1, pf.RB - pf.RB_router - pf.RB_lat, pf.err, lane);
  }
}

// The routing lays out the expert phases: wait for it, copy the tables to
// shared memory and size the rest of the list.
__device__ __forceinline__ void mega_route(const MegaParams& mp, MegaProd& st, VExpert* ve_tab,
                                           int* slot_tab, int lane) {
  const Params& pe = mp.k[KIND_EGU];
  const bool ok = wait_flag(pe.route_ready, pe.err, ERR_WAIT_DEP, lane);
  st.V = 0;
  if (ok) {
    // L2 reads, all in one round trip: the tables and the count were written
    // by another CTA of this launch
    st.V = __ldcg(pe.nve);
    for (int i = lane; i < pe.ve_max; i += 32) {
      const int4 v = __ldcg(reinterpret_cast<const int4*>(pe.ve + i));
      ve_tab[i] = VExpert{v.x, v.y, v.z, v.w};
    }
    for (int i = lane; i < pe.ld_slots; i += 32) slot_tab[i] = __ldcg(pe.slots_sorted + i);
    st.sp[KIND_EGU] = make_space<KIND_EGU>(pe, st.V);
    st.sp[KIND_EDN] = make_space<KIND_EDN>(mp.k[KIND_EDN], st.V);
  } else {
    st.sp[KIND_EGU].total = st.sp[KIND_EDN].total = 0;
    st.sp[KIND_EGU].ppr = st.sp[KIND_EDN].ppr = 1;
  }
  st.sp[KIND_TAIL] = make_space<KIND_TAIL>(mp.k[KIND_TAIL]);
  st.base[KIND_EGU] = mp.n_front;
  st.base[KIND_EDN] = st.base[KIND_EGU] + st.sp[KIND_EGU].total;
  st.base[KIND_TAIL] = st.base[KIND_EDN] + st.sp[KIND_EDN].total;
  st.base[KIND_COUNT] = ok ? st.base[KIND_TAIL] + st.sp[KIND_TAIL].total : mp.n_front;
  st.routed = true;
  __syncwarp();
}

// Kind of list index idx (-1: past the end).  Indices past the front phase
// need the routing; without it they read as "not front" (KIND_EGU).
__device__ __forceinline__ int mega_kind_of(const MegaParams& mp, const MegaProd& st, int idx) {
  if (idx < mp.n_front) return KIND_FRONT;
  if (!st.routed) return KIND_EGU;
  if (idx >= st.base[KIND_COUNT]) return -1;
  if (idx < st.base[KIND_EDN]) return KIND_EGU;
  if (idx < st.base[KIND_TAIL]) return KIND_EDN;
  return KIND_TAIL;
}

// The next list index (grab now unless one is in flight); lane-uniform.
__device__ __forceinline__ int mega_next(MegaProd& st, Ctl* ctl, int workers, int lane) {
  if (!st.in_flight && lane == 0) st.grabbed = atomicAdd(&ctl->cursor, 1) + workers;
  st.in_flight = false;
  return __shfl_sync(0xffffffffu, st.grabbed, 0);
}

template <int KIND>
__device__ __forceinline__ void mega_flush(const MegaParams& mp, MegaProd& st, const int* pend,
                                           int npend, uint8_t* stage_base, const int* slot_tab,
                                           uint64_t* full, int lane) {
  const Params& p = mp.k[KIND];
  mega_wait_deps<KIND>(mp, st, lane);
  st.dep_ok[KIND] = true;
  for (int j = 0; j < npend; ++j) {
    uint8_t* sb = stage_base + (size_t)pend[j] * p.stage_bytes;
    const Hdr& hs = *reinterpret_cast<const Hdr*>(sb);
    issue_act<KIND>(p, hs, sb + p.act_off, &full[pend[j]], lane, slot_tab);
  }
}

// Stream every stage of one piece and return the list index that follows it.
// Weight tiles go out at once; activation copies wait until the phase's
// dependency is met (at most one ring of stages holds weights only).  The
// last stage's header names the next piece's kind, so its consumers know
// whether a phase change follows.
template <int KIND>
__device__ __forceinline__ int mega_issue_piece(const MegaParams& mp, MegaProd& st, int local,
                                                uint8_t* stage_base, const VExpert* ve_tab,
                                                const int* slot_tab, uint64_t* full,
                                                uint64_t* empty, int lane, int workers) {
  const Params& p = mp.k[KIND];
  Ctl* ctl = mp.k[KIND_FRONT].ctl;
  Hdr ph;
  piece_header<KIND>(p, st.sp[KIND], local, ph, ve_tab);
  ph.kind = KIND;
  const int pr = local - ph.p0;
  const int c_first = (pr * p.C) / ph.ppr;
  const int c_last = ((pr + 1) * p.C) / ph.ppr;
  int pend[8];
  int npend = 0;
  int next = -1;
  uint8_t* last_sb = nullptr;
  for (int c = c_first; c < c_last; ++c) {
    if (!st.dep_ok[KIND] && npend == p.nstages) {
      mega_flush<KIND>(mp, st, pend, npend, stage_base, slot_tab, full, lane);
      npend = 0;
    }
    if (!mbar_wait_bounded(&empty[st.stage], st.ephase, p.err, ERR_WAIT_EMPTY, 200)) return -1;
    uint8_t* sb = stage_base + (size_t)st.stage * p.stage_bytes;
    Hdr h = ph;
    chunk_header<KIND>(p, c, c_first, c_last, h);
    h.next_kind = KIND;
    const bool last = c == c_last - 1;
    if (last && st.dep_ok[KIND]) {
      // activations go out with this stage: settle the next piece first
      next = mega_next(st, ctl, workers, lane);
      h.next_kind = mega_kind_of(mp, st, next);
    }
    if (lane == 0) stage_begin<KIND>(p, h, sb, &full[st.stage]);
    __syncwarp();
    if (st.dep_ok[KIND])
      issue_act<KIND>(p, h, sb + p.act_off, &full[st.stage], lane, slot_tab);
    else
      pend[npend++] = st.stage;
    if (last) last_sb = sb;
    if (++st.stage == p.nstages) {
      st.stage = 0;
      st.ephase ^= 1;
    }
  }
  if (!st.dep_ok[KIND]) {
    // the last stage still waits for its activations, so its header can be
    // completed now: no further piece is taken before the dependency resolves
    mega_wait_deps<KIND>(mp, st, lane);
    next = mega_next(st, ctl, workers, lane);
    if (lane == 0 && last_sb) reinterpret_cast<Hdr*>(last_sb)->next_kind = mega_kind_of(mp, st, next);
    __syncwarp();
    st.dep_ok[KIND] = true;
    for (int j = 0; j < npend; ++j) {
      uint8_t* sb = stage_base + (size_t)pend[j] * p.stage_bytes;
      const Hdr& hs = *reinterpret_cast<const Hdr*>(sb);
      issue_act<KIND>(p, hs, sb + p.act_off, &full[pend[j]], lane, slot_tab);
    }
  }
  return next;
}

__device__ void mega_producer(const MegaParams& mp, uint8_t* stage_base, uint8_t* tables,
                              uint64_t* full, uint64_t* empty, int lane) {
  const Params& pf = mp.k[KIND_FRONT];
  Ctl* ctl = pf.ctl;
  VExpert* ve_tab = reinterpret_cast<VExpert*>(tables);
  int* slot_tab = reinterpret_cast<int*>(tables + (size_t)pf.ve_max * sizeof(VExpert));
  MegaProd st;
  st.stage = 0;
  st.ephase = 1;  // empty barriers start "released"
  for (int k = 0; k < KIND_COUNT; ++k) st.dep_ok[k] = false;
  st.routed = false;
  st.V = 0;
  st.sp[KIND_FRONT] = make_space<KIND_FRONT>(pf);
  st.grabbed = 0;
  st.in_flight = false;
  const int workers = (int)gridDim.x - pf.route_cta;
  int idx = blockIdx.x;
  unsigned long long* tr = pf.trace ? pf.trace + (size_t)blockIdx.x * kTraceStride : nullptr;
  while (true) {
    int kind = mega_kind_of(mp, st, idx);
    if (kind != KIND_FRONT && !st.routed) {
      // The routing flag, the tables and the completion counters belong to
      // this forward only once the previous one is over (its last CTA resets
      // them on the way out): a CTA whose first piece is not a front piece
      // must not read any of them before that.
      if (!st.dep_ok[KIND_FRONT]) {
        pdl_wait();
        pdl_trigger();
        st.dep_ok[KIND_FRONT] = true;
      }
      mega_route(mp, st, ve_tab, slot_tab, lane);
      kind = mega_kind_of(mp, st, idx);
    }
    if (kind < 0) break;
    // keep one grab in flight, but only once the previous forward is over
    if (st.dep_ok[KIND_FRONT] && !st.in_flight) {
      if (lane == 0) st.grabbed = atomicAdd(&ctl->cursor, 1) + workers;
      st.in_flight = true;
    }
    if (tr && lane == 0 && tr[8 + kind] == 0) tr[8 + kind] = global_ns();
    switch (kind) {
      case KIND_FRONT:
        idx = mega_issue_piece<KIND_FRONT>(mp, st, idx, stage_base, ve_tab, slot_tab, full, empty, lane, workers);
        break;
      case KIND_EGU:
        idx = mega_issue_piece<KIND_EGU>(mp, st, idx - st.base[KIND_EGU], stage_base, ve_tab, slot_tab, full, empty, lane, workers);
        break;
      case KIND_EDN:
        idx = mega_issue_piece<KIND_EDN>(mp, st, idx - st.base[KIND_EDN], stage_base, ve_tab, slot_tab, full, empty, lane, workers);
        break;
      default:
        idx = mega_issue_piece<KIND_TAIL>(mp, st, idx - st.base[KIND_TAIL], stage_base, ve_tab, slot_tab, full, empty, lane, workers);
        break;
    }
    if (idx < 0) break;
  }
  if (!st.dep_ok[KIND_FRONT]) {  // held no piece at all
    pdl_wait();
    pdl_trigger();
  }
  // end marker
  if (!mbar_wait_bounded(&empty[st.stage], st.ephase, pf.err, ERR_WAIT_EMPTY, 200)) return;
  if (lane == 0) {
    uint8_t* sb = stage_base + (size_t)st.stage * pf.stage_bytes;
    reinterpret_cast<Hdr*>(sb)->flags = HDR_END;
    mbar_arrive(&full[st.stage]);
  }
}

// ---------------------------------------------------------------------------
// consumers

struct MegaCons {
  int stage;
  uint32_t phase;
  int nbuf;
  // split-K ticket in flight (same kind only; settled before a phase change)
  bool pend;
  Hdr pend_h;
  int ticket;
  int tslot;
  bool res_built;
  int n_pieces, n_fin;
};

// One piece of kind KIND whose first stage is full.  Returns false when a
// bounded wait gave up.
template <int KIND, int NT>
__device__ __forceinline__ bool mega_piece(const Params& p, MegaCons& cs, uint8_t* stage_base,
                                           uint64_t* full, uint64_t* empty, uint8_t* scratch,
                                           int* sm_flag, const int* slot_tab, int warp, int lane) {
  const int tid = warp * 32 + lane;
  int* tflag = sm_flag + 4;
  unsigned long long* tr = p.trace ? p.trace + (size_t)blockIdx.x * kTraceStride : nullptr;
  uint8_t* res = stage_base - p.stage_off + p.res_off;
  if (KIND == KIND_TAIL && p.res_off && !cs.res_built) {
    // The resident activation reads y, the combine weights and h_s: acquire
    // the phases that wrote them (the producer has already seen them done).
    if (tid == 0) {
      wait_flag(p.route_ready, p.err, ERR_WAIT_DEP, lane);  // combine weights, nve
      const int V = __ldcg(p.nve);
      wait_count(p.done + 3, V * p.need_rb_edn, p.err, lane);
      wait_count(p.done + 1, p.need_rb_sh, p.err, lane);
    }
    named_sync(1, kConsumerThreads);
    build_resident(p, res, tid, 0, p.res_k);
    named_sync(1, kConsumerThreads);
    cs.res_built = true;
  }
  float acc[NT][4], acc2[NT][4];
  zero_acc(acc);
  zero_acc(acc2);
  Hdr h;
  while (true) {
    uint8_t* sb = stage_base + (size_t)cs.stage * p.stage_bytes;
    h = *reinterpret_cast<const Hdr*>(sb);
    if (tr && tid == 0 && tr[15 + KIND] == 0) tr[15 + KIND] = global_ns();
    const uint8_t* tile = sb + kHdrBytes;
    const uint8_t* act = sb + p.act_off;
    if (KIND == KIND_FRONT) {
      mma_dense_x<NT>(p, h, tile, act, acc, acc2, warp, lane);
    } else if (KIND == KIND_EGU || KIND == KIND_EDN) {
      mma_mx<NT>(p, h, tile, act, acc, warp, lane);
    } else if (p.res_off) {
      mma_tail_resident<NT>(p, h, tile, res, acc, acc2, warp, lane);
    } else {
      uint8_t* tbuf = scratch + 4096 + (cs.nbuf & 1) * (16 * 320);
      ++cs.nbuf;
      mma_tail<NT>(p, h, tile, act, tbuf, acc, acc2, warp, lane, tid);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[cs.stage]);
    if (++cs.stage == p.nstages) {
      cs.stage = 0;
      cs.phase ^= 1;
    }
    if (h.flags & HDR_LAST) break;
    if (!mbar_wait_bounded(&full[cs.stage], cs.phase, p.err, ERR_WAIT_FULL)) return false;
  }
  ++cs.n_pieces;
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[t][q] += acc2[t][q];
  // settle every ticket now when the phase changes next (a later phase may
  // wait for what it finalises) and for router row blocks (the routing waits
  // for them)
  const bool settle = h.next_kind != KIND || (KIND == KIND_FRONT && h.rb < p.RB_router);
  if (h.ppr == 1) {
    if (cs.pend && settle) {
      if (tid == 0) tflag[cs.tslot] = (cs.ticket == cs.pend_h.ppr - 1);
      named_sync(1, kConsumerThreads);
      const bool fin = tflag[cs.tslot] != 0;
      const Hdr prev = cs.pend_h;
      cs.pend = false;
      cs.tslot ^= 1;
      // (acc still holds this piece; finalise the earlier one after it)
      ++cs.n_fin;
      epilogue<KIND, NT>(p, h, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
      if (fin) {
        ++cs.n_fin;
        finalize<KIND, NT>(p, prev, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
      }
      return true;
    }
    ++cs.n_fin;
    epilogue<KIND, NT>(p, h, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
    return true;
  }
  write_partial<NT>(p, h.piece, h.ntok, acc, warp, lane);
  if (settle) {
    if (tid == 0) {
      if (cs.pend) tflag[cs.tslot] = (cs.ticket == cs.pend_h.ppr - 1);
      sm_flag[6] = (atom_add_acqrel(p.counters + h.v * p.RB + h.rb, 1) == h.ppr - 1);
    }
    named_sync(1, kConsumerThreads);
    const bool fin_prev = cs.pend && tflag[cs.tslot] != 0;
    const bool fin_now = sm_flag[6] != 0;
    const Hdr prev = cs.pend_h;
    cs.pend = false;
    cs.tslot ^= 1;
    named_sync(1, kConsumerThreads);  // flags read before they are reused
    if (fin_prev) {
      ++cs.n_fin;
      finalize<KIND, NT>(p, prev, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
    }
    if (fin_now) {
      ++cs.n_fin;
      const unsigned long long t0 = tr ? global_ns() : 0ull;
      finalize<KIND, NT>(p, h, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
      if (tr && tid == 0) tr[7] += global_ns() - t0;
    }
    return true;
  }
  // same phase follows: read this ticket one piece later
  if (tid == 0 && cs.pend) tflag[cs.tslot] = (cs.ticket == cs.pend_h.ppr - 1);
  named_sync(1, kConsumerThreads);  // every warp's partials precede thread 0's release
  const bool fin = cs.pend && tflag[cs.tslot] != 0;
  if (tid == 0) cs.ticket = atom_add_acqrel(p.counters + h.v * p.RB + h.rb, 1);
  const Hdr prev = cs.pend_h;
  cs.pend_h = h;
  cs.pend = true;
  cs.tslot ^= 1;
  if (fin) {
    ++cs.n_fin;
    finalize<KIND, NT>(p, prev, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
  }
  return true;
}

// A ticket still deferred when the stream ends (a resident-tail stage carries
// no activation bytes, so it can complete before its header learns that no
// piece follows): settle it.
template <int KIND, int NT>
__device__ __forceinline__ void mega_settle_pending(const Params& p, MegaCons& cs, uint8_t* scratch,
                                                    int* sm_flag, const int* slot_tab, int warp,
                                                    int lane) {
  const int tid = warp * 32 + lane;
  int* tflag = sm_flag + 4;
  if (tid == 0) tflag[cs.tslot] = (cs.ticket == cs.pend_h.ppr - 1);
  named_sync(1, kConsumerThreads);
  const bool fin = tflag[cs.tslot] != 0;
  const Hdr prev = cs.pend_h;
  cs.pend = false;
  cs.tslot ^= 1;
  if (fin) {
    float acc[NT][4];
    ++cs.n_fin;
    finalize<KIND, NT>(p, prev, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
  }
}

template <int NT>
__device__ void mega_consumer(const MegaParams& mp, uint8_t* stage_base, uint64_t* full,
                              uint64_t* empty, uint8_t* scratch, int* sm_flag, const int* slot_tab,
                              int warp, int lane) {
  const Params& pf = mp.k[KIND_FRONT];
  const int tid = warp * 32 + lane;
  // activations and partial sums of the previous forward are read only
  // after it is over
  pdl_wait();
  pdl_trigger();
  MegaCons cs;
  cs.stage = 0;
  cs.phase = 0;
  cs.nbuf = 0;
  cs.pend = false;
  cs.ticket = 0;
  cs.tslot = 0;
  cs.res_built = false;
  cs.n_pieces = cs.n_fin = 0;
  bool ok = true;
  while (ok) {
    if (!mbar_wait_bounded(&full[cs.stage], cs.phase, pf.err, ERR_WAIT_FULL)) break;
    const Hdr& h = *reinterpret_cast<const Hdr*>(stage_base + (size_t)cs.stage * pf.stage_bytes);
    const int flags = h.flags, kind = h.kind;
    if (flags & HDR_END) {
      if (cs.pend) {
        switch (cs.pend_h.kind) {
          case KIND_FRONT: mega_settle_pending<KIND_FRONT, NT>(mp.k[KIND_FRONT], cs, scratch, sm_flag, slot_tab, warp, lane); break;
          case KIND_EGU: mega_settle_pending<KIND_EGU, NT>(mp.k[KIND_EGU], cs, scratch, sm_flag, slot_tab, warp, lane); break;
          case KIND_EDN: mega_settle_pending<KIND_EDN, NT>(mp.k[KIND_EDN], cs, scratch, sm_flag, slot_tab, warp, lane); break;
          default: mega_settle_pending<KIND_TAIL, NT>(mp.k[KIND_TAIL], cs, scratch, sm_flag, slot_tab, warp, lane); break;
        }
      }
      break;
    }
    switch (kind) {
      case KIND_FRONT:
        ok = mega_piece<KIND_FRONT, NT>(mp.k[KIND_FRONT], cs, stage_base, full, empty, scratch, sm_flag, slot_tab, warp, lane);
        break;
      case KIND_EGU:
        ok = mega_piece<KIND_EGU, NT>(mp.k[KIND_EGU], cs, stage_base, full, empty, scratch, sm_flag, slot_tab, warp, lane);
        break;
      case KIND_EDN:
        ok = mega_piece<KIND_EDN, NT>(mp.k[KIND_EDN], cs, stage_base, full, empty, scratch, sm_flag, slot_tab, warp, lane);
        break;
      default:
        ok = mega_piece<KIND_TAIL, NT>(mp.k[KIND_TAIL], cs, stage_base, full, empty, scratch, sm_flag, slot_tab, warp, lane);
        break;
    }
  }
  if (pf.trace && tid == 0) {
    unsigned long long* tr = pf.trace + (size_t)blockIdx.x * kTraceStride;
    tr[2] = (unsigned long long)cs.n_pieces;
    tr[3] = (unsigned long long)cs.n_fin;
  }
}

// ---------------------------------------------------------------------------

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) moe_mega_kernel(const __grid_constant__ MegaParams mp) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const Params& pf = mp.k[KIND_FRONT];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  int* sm_flag = reinterpret_cast<int*>(smem + 256);
  uint8_t* scratch = smem + pf.scratch_off;
  uint8_t* stages = smem + pf.stage_off;
  uint8_t* tables = smem + pf.table_off;
  const int* slot_tab = reinterpret_cast<const int*>(tables + (size_t)pf.ve_max * sizeof(VExpert));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (pf.trace && threadIdx.x == 0) {
    unsigned long long* tr = pf.trace + (size_t)blockIdx.x * kTraceStride;
    tr[0] = global_ns();
    for (int i = 2; i < kTraceStride; ++i) tr[i] = 0;
    tr[14] = smid();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < pf.nstages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (blockIdx.x == gridDim.x - 1) {
    // the routing CTA: it writes the routing tables the previous forward read
    pdl_wait();
    pdl_trigger();
    if (warp < kConsumerWarps)
      route_cta(pf, scratch, reinterpret_cast<float*>(stages), sm_flag, threadIdx.x, warp, lane,
                8 * kRowsPerBlock);
  } else if (warp == kConsumerWarps) {
    mega_producer(mp, stages, tables, full, empty, lane);
  } else {
    mega_consumer<NT>(mp, stages, full, empty, scratch, sm_flag, slot_tab, warp, lane);
  }
  __syncthreads();
  if (pf.trace && threadIdx.x == 0) pf.trace[(size_t)blockIdx.x * kTraceStride + 1] = global_ns();
  if (threadIdx.x == 0) {
    Ctl* ctl = pf.ctl;
    __threadfence();
    if (atomicAdd(&ctl->exits, 1) == (int)gridDim.x - 1) {
      // last CTA out: every reader of the counters and flags has left
      ctl->cursor = 0;
      ctl->exits = 0;
      for (int i = 0; i < 4; ++i) pf.done[i] = 0;
      *pf.route_ready = 0;
      __threadfence();
    }
  }
}

template <int NT>
static int launch_mega_nt(const MegaParams& mp, int grid, size_t smem, cudaStream_t s, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return (int)cudaLaunchKernelEx(&cfg, moe_mega_kernel<NT>, mp);
}

}  // namespace moe
