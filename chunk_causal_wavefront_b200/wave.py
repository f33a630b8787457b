"""Wave Parallelism delivery plan: which rank sends which slot's K/V to whom.

"Wave Forcing: Towards Speed-of-Light Streaming Video Generation", Method
section and Figure 3c: each denoising stage (and the store) runs on its own
GPU, one chunk per round, and publishes its chunk's K/V directly into the
attention slots of the stages that read them, followed by a ready signal; K/V
flow one way (thelatestinai listing, Table 10: no reverse edge).

Rank r owns slot r (r = 0..S, the store is slot S), so the world has S + 1
ranks. In round k slot s is live iff k - s >= 0. Under the WF mask slot s reads
slots j >= s; so slot j's pages go to every live slot s < j. Under the RF mask
every live slot reads every other. The store's chunk becomes the anchor or a
history chunk of every later round, so it goes to every rank, live or not.

The plan is host logic only: each rank computes the same plan from (S, k,
mask) with no communication, and calls wf_deliver_kv for its own slot's
entries.

Ordering is the caller's: a receiver may run its round-k attention only after
every round-k delivery into its pool has landed, and a sender must not deliver
round k + 1 into a receiver until that receiver's round-k attention has
finished reading its pages, since the delivery overwrites the same pages (and
the recycled store pages) in place. A barrier after each round's attention, or
an event the receiver records after it and the sender waits for, gives that
order; the readiness check reads the ready tags once, when the attention kernel
starts, so it cannot catch an overwrite that lands while the kernel runs."""
from typing import Dict, List


def live_slots(num_stages: int, k: int) -> List[int]:
    """Live query slots of round k (denoising slots 0..S-1, then the store S)."""
    S = num_stages
    return [s for s in range(S) if k - s >= 0] + ([S] if k >= S else [])


def readers(num_stages: int, k: int, slot: int, mask: str = "wf") -> List[int]:
    """Ranks, other than the owner, that need `slot`'s K/V of round k."""
    S = num_stages
    live = live_slots(S, k)
    if slot not in live:
        return []
    if slot == S:
        return [r for r in range(S + 1) if r != S]
    if mask == "rf":
        return [s for s in live if s != slot]
    if mask != "wf":
        raise ValueError(f"unknown mask {mask!r}")
    return [s for s in live if s < slot]


def wave_plan(num_stages: int, k: int, mask: str = "wf") -> Dict[int, List[int]]:
    """{slot: receiver ranks} for every live slot of round k."""
    return {j: readers(num_stages, k, j, mask) for j in live_slots(num_stages, k)}
