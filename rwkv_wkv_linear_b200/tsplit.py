"""One sequence split over T across ranks: the one exchange of the WKV state.

The WKV state is a sequence's whole history ("An RNN that claims to match
transformers, now in chatbot form", "The interesting bit"), and one segment's
state from the empty state combines with the state before it by a closed
form (wkv4_state_combine).  So a long sequence can be cut into consecutive
segments, one per rank in rank order, and run as:

  1. summary    every rank runs the forward over its own segment from the
                empty state and keeps only the final state S_r;
  2. exchange   all-gather of every rank's S_r ([3, B, C] fp32, 12 bytes a
                channel) and segment length T_r over the process group (a
                plain NCCL or gloo collective);
  3. combine    rank r joins the sequence's initial state with S_0 .. S_{r-1}
                in order (on the device): the state entering its segment;
  4. recompute  the forward over its segment from that state gives the
                segment's outputs and final state; the last rank's final
                state is the whole sequence's.

Every step runs in the library's kernels (wkv4.forward, wkv4.state_combine);
this module only orders them and moves the [3, B, C] summaries.  k and v are
read twice (summary and recompute), the price of the split.  The arithmetic
steps are passed in as an `ops` object so that the rank logic can be checked
on CPU processes against other implementations of them.
"""

from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


class DeviceOps:
    """The library's kernels (CUDA tensors)."""

    def forward(self, k, v, w, u, state_in):
        from rwkv_wkv_linear_b200 import wkv4
        return wkv4.forward(k, v, w, u, state_in)

    def combine(self, x, y, n_steps: int, w):
        from rwkv_wkv_linear_b200 import wkv4
        return wkv4.state_combine(x, y, n_steps, w)


def segment_prefixes(summaries: Sequence[torch.Tensor], lengths: Sequence[int], w: torch.Tensor,
                     state_in: Optional[torch.Tensor], ops, upto: Optional[int] = None
                     ) -> List[Optional[torch.Tensor]]:
    """The state entering each segment (step 3): prefixes[r] = state_in
    followed by segments 0 .. r-1 (None stands for the empty state), for
    r = 0 .. upto (default: every segment)."""
    upto = len(summaries) - 1 if upto is None else upto
    prefixes = [state_in]
    for q in range(upto):
        prefixes.append(ops.combine(prefixes[-1], summaries[q], int(lengths[q]), w))
    return prefixes


def forward_tsplit(k: torch.Tensor, v: torch.Tensor, w: torch.Tensor, u: torch.Tensor,
                   state_in: Optional[torch.Tensor] = None, *, group=None,
                   ops=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's segment of a sequence split over T across the ranks of
    `group` (segments in rank order; k, v [B, T_r, C]; w, u [C]; state_in
    [3, B, C] the sequence's initial state, the same on every rank, or None).
    Returns (y [B, T_r, C], the state after this segment).  Every rank takes
    part in the two all-gathers, in the same order."""
    ops = ops or DeviceOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    _, summary = ops.forward(k, v, w, u, None)
    summary = summary.contiguous()
    gathered = [torch.empty_like(summary) for _ in range(world)]
    dist.all_gather(gathered, summary, group=group)
    length = torch.tensor([k.shape[1]], dtype=torch.int64, device=summary.device)
    lengths = [torch.empty_like(length) for _ in range(world)]
    dist.all_gather(lengths, length, group=group)
    lens = [int(t.item()) for t in lengths]
    prefix = segment_prefixes(gathered, lens, w, state_in, ops, upto=rank)[rank]
    return ops.forward(k, v, w, u, prefix)
