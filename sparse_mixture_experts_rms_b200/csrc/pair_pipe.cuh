// pair_pipe.cuh -- the producer's end of the operand pipeline shared by the
// 2-CTA (cta_group::2) grouped GEMMs (bf16 and MXFP8).
//
// Each pipeline stage is loaded half by each CTA of the pair, and both halves
// complete on the pair leader's "full" barrier of the stage, which the
// leader's producer arms with the bytes of both halves.  A CTA must not exit
// while a copy into its shared memory is in flight.  When a bounded wait gives
// up somewhere in the pair, the two producers may stop after different
// stages, and a stage that only one of them issued can never complete as
// armed; the peer cannot observe its own copies at all (they signal the
// leader's barrier).  So at the end each producer reports how many stages it
// issued, and the leader settles the accounting of the stages only one side
// issued, waits until every stage in flight has landed, and releases the
// peer.  These waits keep the default limit: copies already issued always
// finish.
#pragma once

#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {

// In each CTA's shared memory (the leader's `hs` and `issued`, the peer's
// `landed` are the ones used).
struct PairDrain {
  uint64_t hs;         // leader: both producers have stopped issuing (2 arrivals)
  uint64_t landed;     // peer: every stage issued by either producer has landed
  uint32_t issued[2];  // leader: stages issued by the leader / by the peer
};

__device__ __forceinline__ void pair_drain_init(PairDrain& pd) {
  mbar_init(&pd.hs, 2);
  mbar_init(&pd.landed, 1);
}

// Called once by each CTA's producer thread after its last issue (the end of
// its tile list, or earlier when a wait gave up), with the number of stages it
// issued.  `full` = this CTA's full barriers (used on the leader), `half_tx` =
// the bytes one CTA loads per stage (the two halves are the same size).
//
// A stage j is issued only after stage j - STAGES was consumed, which needs
// both halves of it; so the two counts differ by at most STAGES, stages below
// max(counts) - STAGES have landed, and each barrier of the last STAGES
// stages is in the phase of the one stage that uses it.  For a stage only the
// peer issued, the leader arrives expecting the peer's half; for a stage only
// the leader issued, it retires the peer's missing half (complete_tx).  Then
// every phase of the last STAGES stages completes once its copies have landed.
template <int STAGES>
__device__ void pair_producer_drain(PairDrain& pd, uint64_t* full, uint32_t issued, uint32_t rank,
                                    uint32_t half_tx, uint32_t* err) {
  volatile int no_abort = 0;
  if (rank != 0) {
    st_cluster_u32(map_to_cta(smem_addr(&pd.issued[1]), 0), issued);
    mbar_arrive_cluster(map_to_cta(smem_addr(&pd.hs), 0));  // release: the count is visible first
    mbar_wait(&pd.landed, 0, &no_abort, err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs, true);
    return;
  }
  pd.issued[0] = issued;
  mbar_arrive(&pd.hs);
  uint32_t peer = issued;  // if the peer never reports, settle nothing
  if (mbar_wait(&pd.hs, 0, &no_abort, err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs, true))
    peer = *reinterpret_cast<volatile uint32_t*>(&pd.issued[1]);
  const uint32_t hi = issued > peer ? issued : peer;
  const uint32_t lo = issued < peer ? issued : peer;
  for (uint32_t j = lo; j < hi; ++j) {
    uint64_t* b = &full[j % STAGES];
    if (j >= issued)
      mbar_arrive_expect_tx(b, half_tx);  // only the peer issued stage j
    else
      mbar_complete_tx(b, half_tx);       // only the leader issued stage j
  }
  for (uint32_t j = hi > STAGES ? hi - STAGES : 0; j < hi; ++j)
    mbar_wait(&full[j % STAGES], (j / STAGES) & 1u, &no_abort, err, MOE_DEVERR_TIMEOUT, kWaitTimeoutNs);
  mbar_arrive_cluster(map_to_cta(smem_addr(&pd.landed), 1));
}

}  // namespace moe
