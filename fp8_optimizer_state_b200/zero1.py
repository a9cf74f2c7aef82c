"""ZeRO-1 data parallelism around the FP8-state AdamW step.

COAT's memory figures ("FP8训练新范式：减少40%显存占用，训练速度提高1.4倍",
section 训练加速1.43倍，显存降低1.54倍) are per GPU of a four-GPU training run;
the page does not say how the run is parallelised.  Under data parallelism
the optimizer states need only be kept once across the GPUs: here each of
world_size ranks keeps the FP32 master weights and the FP8 moments (codes,
root scales, k) of 1/world_size of all parameter groups, as
coat_zero1_layout partitions them, and every rank keeps the whole bf16
weight copy and a whole gradient buffer.  One step:

  1. a reduce-scatter (sum over ranks) of the flat bf16 gradient buffer, so
     that each rank receives the summed gradients of its own groups;
  2. the multi-tensor FP8 AdamW step (coat_adamw_step_multi) over the rank's
     pieces, writing their bf16 weights into the rank's weight shard;
  3. an all-gather of the weight shards into every rank's flat bf16 weights.

The collectives are torch.distributed calls (NCCL over NVLink / NVSwitch on
B200s); the step is the library's kernel and no arithmetic of the step runs
here.  Gradients are summed, not averaged: scale the loss by 1/world_size for
their mean.  Groups never span ranks, so the result is the single-GPU step on
the summed gradients, bit for bit.

The sum itself is taken in bf16 by the collective, which may round after each
of its world_size - 1 additions: an element of the summed gradient is within
(world_size - 1) u (1 + world_size u) sum_r |g_r| of the exact sum (u = 2^-8,
bf16's unit roundoff; each partial sum is at most sum_r |g_r|).  That is the
only difference from a step on the exact sum of the ranks' gradients
(tests/test_zero1_cpu.py checks the bound at 2, 4 and 8 ranks).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (COAT_E4M3, GROUP, coat_adamw_step_multi, coat_adamw_step_multi_clipped,
               coat_grad_clip_finalize, coat_multi_plan_create, coat_zero1_layout, make_desc,
               new_grad_clip)


class Zero1AdamW:
    """ZeRO-1 sharded AdamW over FP8 moments for tensors of `sizes` elements.

    Buffers on `device`:
      flat_grad    flat_elems bf16: tensor i's gradient is grad(i), written by
                   the caller before step(); the padding stays zero.
      flat_weight  flat_elems bf16: tensor i's bf16 weights are weight(i),
                   complete on every rank after step().
      grad_shard, weight_shard: this rank's slices of the flat buffers
                   (shard_elems each, starting at rank * shard_elems).
      master, m_q, v_q: shard_elems each (FP32, u8, u8); m_scale, m_k,
                   v_scale, v_k: one float per group of the shard.  Moments
                   start at zero (codes 0, scale 1, k 1).
    Per rank: 4 bytes per parameter for the two flat bf16 buffers, and
    6.125 / world_size for the sharded state (master 4, codes 2, scale and k
    16 per group of 128).
    The process group's collectives must support bf16 reduce-scatter and
    all-gather (NCCL; gloo on the CPU)."""

    def __init__(self, sizes, *, device, process_group=None, fmt_m=COAT_E4M3, fmt_v=COAT_E4M3):
        self.pg = process_group
        self.world = dist.get_world_size(process_group)
        self.rank = dist.get_rank(process_group)
        self.sizes = [int(x) for x in sizes]
        self.pieces, self.shard_elems, self.flat_elems, self.flat_offsets = coat_zero1_layout(
            self.sizes, self.world, self.rank)
        self.fmt_m, self.fmt_v = fmt_m, fmt_v
        dev = torch.device(device)
        e, ng = self.shard_elems, self.shard_elems // GROUP
        bf16 = dict(dtype=torch.bfloat16, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.flat_grad = torch.zeros(self.flat_elems, **bf16)
        self.flat_weight = torch.zeros(self.flat_elems, **bf16)
        # The rank's shards are its slices of the flat buffers: the
        # reduce-scatter and the all-gather then run in place (NCCL's in-place
        # forms), and no second copy of either is held.
        lo = self.rank * e
        self.grad_shard = self.flat_grad[lo:lo + e]
        self.weight_shard = self.flat_weight[lo:lo + e]
        self.master = torch.zeros(e, **f32)
        self.m_q = torch.zeros(e, dtype=torch.uint8, device=dev)
        self.v_q = torch.zeros(e, dtype=torch.uint8, device=dev)
        self.m_scale, self.m_k, self.v_scale, self.v_k = (torch.ones(ng, **f32) for _ in range(4))
        self._plan = None
        self._wd_scale = None
        # clip record (24 bytes): its first double, the sum of squares, is
        # all-reduced over the ranks
        self.clip = new_grad_clip(dev)
        self.clip_sumsq = self.clip[:8].view(torch.float64)

    # -- views ------------------------------------------------------------
    def grad(self, i):
        """Tensor i's gradient in the flat gradient buffer (a 1-D view)."""
        o = self.flat_offsets[i]
        return self.flat_grad[o:o + self.sizes[i]]

    def weight(self, i):
        """Tensor i's bf16 weights in the flat weight buffer (a 1-D view)."""
        o = self.flat_offsets[i]
        return self.flat_weight[o:o + self.sizes[i]]

    def piece_views(self, piece):
        """The shard's slices for one piece, as the step reads and writes them:
        master, weight, grad (n elements), m_q / v_q (whole groups) and the
        four per-group metadata slices."""
        _, _, n, sb = piece
        g0, ng = sb // GROUP, -(-n // GROUP)
        return dict(master=self.master[sb:sb + n], weight=self.weight_shard[sb:sb + n],
                    grad=self.grad_shard[sb:sb + n],
                    m_q=self.m_q[sb:sb + ng * GROUP], m_scale=self.m_scale[g0:g0 + ng],
                    m_k=self.m_k[g0:g0 + ng], v_q=self.v_q[sb:sb + ng * GROUP],
                    v_scale=self.v_scale[g0:g0 + ng], v_k=self.v_k[g0:g0 + ng])

    # -- state ------------------------------------------------------------
    def load_weights(self, tensors):
        """Set the master weights of this rank's pieces and the whole bf16
        copy from full-precision `tensors` (one per size, any shape)."""
        if len(tensors) != len(self.sizes):
            raise ValueError("need one tensor per size (%d), got %d"
                             % (len(self.sizes), len(tensors)))
        for i, t in enumerate(tensors):
            flat = t.detach().reshape(-1)
            if flat.numel() != self.sizes[i]:
                raise ValueError("tensor %d has %d elements, expected %d"
                                 % (i, flat.numel(), self.sizes[i]))
            self.weight(i).copy_(flat.to(torch.float32).to(torch.bfloat16))
        for piece in self.pieces:
            t, b, n, _ = piece
            self.piece_views(piece)["master"].copy_(
                tensors[t].detach().reshape(-1)[b:b + n].to(torch.float32))

    def set_wd_scale(self, scales):
        """Per-tensor weight decay multipliers (one per size; e.g. 0 for
        normalisation weights), applied from the next step."""
        if len(scales) != len(self.sizes):
            raise ValueError("need one scale per tensor")
        self._wd_scale = [float(scales[t]) for t, _, _, _ in self.pieces]
        if self._plan is not None:
            self._plan.set_wd_scale(self._wd_scale)

    _STATE = ("master", "m_q", "m_scale", "m_k", "v_q", "v_scale", "v_k")

    def state_dict(self):
        """This rank's optimizer state (CPU copies): the shard's master
        weights and FP8 moments, with the layout they belong to."""
        out = {k: getattr(self, k).detach().cpu().clone() for k in self._STATE}
        out.update(sizes=list(self.sizes), world_size=self.world, rank=self.rank,
                   fmt_m=self.fmt_m, fmt_v=self.fmt_v)
        return out

    def load_state_dict(self, state):
        """Restore this rank's state saved by state_dict() under the same
        sizes, world size, rank and formats, then rebuild the bf16 weights:
        each piece's bf16 copy is RNE(master), as the step writes it, and the
        weights are all-gathered (a collective: every rank calls this)."""
        want = dict(sizes=self.sizes, world_size=self.world, rank=self.rank, fmt_m=self.fmt_m,
                    fmt_v=self.fmt_v)
        got = {k: state[k] for k in want}
        if got != want:
            raise ValueError("state was saved under another layout: %r, expected %r"
                             % (got, want))
        for k in self._STATE:
            dst = getattr(self, k)
            src = state[k]
            if src.dtype != dst.dtype or src.shape != dst.shape:
                raise ValueError("state %s has %s %s, expected %s %s"
                                 % (k, src.dtype, tuple(src.shape), dst.dtype, tuple(dst.shape)))
            dst.copy_(src)
        for piece in self.pieces:
            v = self.piece_views(piece)
            v["weight"].copy_(v["master"].to(torch.bfloat16))
        self.all_gather_weights()

    # -- the step ---------------------------------------------------------
    def reduce_scatter_grads(self, async_op=False):
        """Sum the ranks' flat gradients into this rank's shard (in place).
        async_op: return the collective's work handle instead of waiting, so
        that the caller can overlap it (wait() before the norm pass or step)."""
        return dist.reduce_scatter_tensor(self.grad_shard, self.flat_grad,
                                          op=dist.ReduceOp.SUM, group=self.pg,
                                          async_op=async_op)

    def _get_plan(self, stream=None):
        if self._plan is None:
            descs = []
            for piece in self.pieces:
                v = self.piece_views(piece)
                descs.append(make_desc(v["master"], v["weight"], v["grad"], v["m_q"],
                                       v["m_scale"], v["m_k"], v["v_q"], v["v_scale"], v["v_k"]))
            self._plan = coat_multi_plan_create(descs, self.fmt_m, self.fmt_v, stream=stream)
            if self._wd_scale is not None:
                self._plan.set_wd_scale(self._wd_scale, stream=stream)
        return self._plan

    def local_grad_sumsq(self):
        """This rank's sum of squared summed gradients into the clip record
        (the gradient-norm pass over the rank's pieces; 0 without pieces)."""
        if self.pieces:
            self._get_plan().grad_norm(float("inf"), self.clip)
        else:
            self.clip.zero_()

    def allreduce_grad_sumsq(self):
        dist.all_reduce(self.clip_sumsq, op=dist.ReduceOp.SUM, group=self.pg)

    def finalize_clip(self, max_norm):
        """Norm, coefficient and found-Inf from the global sum of squares."""
        coat_grad_clip_finalize(self.clip, max_norm)

    def local_step(self, *, lr, beta1, beta2, eps, wd, step, clipped=False, stream=None):
        """The FP8 AdamW step over this rank's pieces (one kernel launch);
        clipped: scale the gradients by the clip record's coefficient, or
        skip the step when it found an Inf or NaN."""
        if not self.pieces:
            return
        plan = self._get_plan(stream)
        if clipped:
            coat_adamw_step_multi_clipped(plan, self.clip, lr=lr, beta1=beta1, beta2=beta2,
                                          eps=eps, wd=wd, step=step, stream=stream)
        else:
            coat_adamw_step_multi(plan, lr=lr, beta1=beta1, beta2=beta2, eps=eps, wd=wd,
                                  step=step, stream=stream)

    def all_gather_weights(self, async_op=False):
        """Gather every rank's bf16 weight shard into the flat weights (in
        place).  async_op: return the work handle, e.g. to overlap the gather
        with work that does not read the weights; wait() before reading them."""
        return dist.all_gather_into_tensor(self.flat_weight, self.weight_shard, group=self.pg,
                                           async_op=async_op)

    def step(self, *, lr, beta1, beta2, eps, wd, step, max_norm=None):
        """Reduce-scatter the gradients, step this rank's share, all-gather
        the bf16 weights.  With max_norm, the summed gradients are clipped to
        that global 2-norm first (the norm over all ranks' shards: each rank's
        sum of squares, all-reduced, then the coefficient on the device), and
        an Inf or NaN anywhere skips the step on every rank."""
        self.reduce_scatter_grads()
        if max_norm is not None:
            self.local_grad_sumsq()
            self.allreduce_grad_sumsq()
            self.finalize_clip(max_norm)
        self.local_step(lr=lr, beta1=beta1, beta2=beta2, eps=eps, wd=wd, step=step,
                        clipped=max_norm is not None)
        self.all_gather_weights()

    def close(self):
        if self._plan is not None:
            self._plan.destroy()
            self._plan = None
