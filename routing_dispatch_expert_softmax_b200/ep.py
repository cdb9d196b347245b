"""Expert parallelism across ranks: ``EPMoELayer``.

The exchange the pages centre on ("Serving MoE models with expert parallelism
on 8xH200", section "Tensor parallel vs expert parallel"; "Wide Expert
Parallelism", section "All-to-all communication: the essential tradeoff";
"Expert Parallelism for MoE Models", section "Mechanics of Token Routing and
All-to-All Communication"): R ranks, one process per GPU, each holding E/R
whole experts (rank r owns experts [r*E/R, (r+1)*E/R), the contiguous
placement of "Wide Expert Parallelism", section "Expert Parallelism: keep
specialists whole") and its own tokens.  A layer call on every rank:

1. router and top-k over all E experts for the rank's own tokens
   (``moe_router`` + ``moe_topk``);
2. dispatch with ``R`` virtual ranks (``moe_dispatch``): the expert-major
   buffer is then rank-contiguous, the slice for rank r ordered by r's local
   expert;
3. all-to-all of the per-expert row counts, then all-to-all-v of the row
   slices (NCCL through ``torch.distributed``);
4. on the receiving rank: each received row labelled with its local expert
   (``moe_ep_recv_experts``), regrouped expert-major across sources
   (``moe_dispatch`` with k = 1), the local experts' SwiGLU FFNs
   (``moe_ffn``), and the rows put back in received order (``moe_combine``
   with k = 1 and unit gates, an exact copy);
5. the reverse all-to-all-v returns each row to its source, which sums its
   tokens' k rows with the gates (``moe_combine``).

Every step of the arithmetic runs in the library's kernels; torch supplies
device memory, streams and the collectives.  The split sizes of an
all-to-all-v must be known on the host, so each call synchronises once on
the exchanged counts.  Weights never move; no TMA or library GEMM ever reads
a peer's memory (the exchanged rows land in this GPU's memory first).

The phases are separate methods so the same arithmetic can be driven by any
exchange: ``forward`` uses a communicator over ``torch.distributed``; a
caller (or a test) holding all ranks' states in one process can run the
phases itself.  ``ops`` (default: the C ABI) is the per-step arithmetic.
"""

from __future__ import annotations

from typing import List, Optional

import torch

from . import binding as B


class LibraryOps:
    """The per-step arithmetic of the expert-parallel layer, through the C ABI
    (device tensors; no CPU path)."""

    def __init__(self):
        B.load_library()
        self._ws: Optional[torch.Tensor] = None

    def _workspace(self, shape: B.MoEShape, device) -> torch.Tensor:
        """One workspace for every call of this rank (they run in order on
        one stream), grown when a call needs more; the received row count
        changes from call to call, so a workspace per shape would pile up."""
        need = B.moe_workspace_size(shape)
        if need == 0:
            raise B.MoEError(B.MOE_ERR_INVALID_ARG, "moe_workspace_size")
        if self._ws is None or self._ws.numel() < need or self._ws.device != torch.device(device):
            self._ws = B.workspace(shape, device)
        return self._ws

    def route(self, x, w_g, bias, k: int, f: int):
        T, d = x.shape
        E = w_g.shape[1]
        shape = B.MoEShape.of(T, d, E, k, f)
        ws = self._workspace(shape, x.device)
        logits = torch.empty(T, E, dtype=torch.float32, device=x.device)
        idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
        w = torch.empty(T, k, dtype=torch.float32, device=x.device)
        if T:
            B.moe_router(x, w_g, bias, logits, shape, ws)
            B.moe_topk(logits, idx, w, shape)
        return idx, w

    def dispatch(self, idx, x, E: int, R: int, f: int):
        T, k = idx.shape
        d = x.shape[1]
        dev = x.device
        shape = B.MoEShape.of(T, d, E, k, f, R if R > 1 else 0)
        ws = self._workspace(shape, dev)
        i32 = lambda *n: torch.empty(*n, dtype=torch.int32, device=dev)
        out = dict(counts=i32(E), offsets=i32(E + 1), perm=i32(T * k), row_of=i32(T, k),
                   x_perm=torch.empty(T * k, d, dtype=x.dtype, device=dev),
                   rank_offsets=i32(R + 1) if R > 1 else None)
        B.moe_dispatch(idx if T else None, x if T else None, out["counts"], out["offsets"],
                       out["perm"] if T else None, out["row_of"] if T else None,
                       out["x_perm"] if T else None, shape, ws, None, out["rank_offsets"])
        out["status"] = ws
        return out

    def recv_experts(self, recv_counts, R: int, E_loc: int, N: int):
        out = torch.empty(N, dtype=torch.int32, device=recv_counts.device)
        if N:
            B.moe_ep_recv_experts(recv_counts, R, E_loc, N, out)
        return out

    def ffn(self, x_em, offsets, w13, w2, E_loc: int):
        N, d = x_em.shape
        f = w2.shape[2]
        z = torch.empty(N, d, dtype=torch.bfloat16, device=x_em.device)
        if N:
            shape = B.MoEShape.of(N, d, E_loc, 1, f)
            B.moe_ffn(x_em, offsets, w13, w2, z, shape, self._workspace(shape, x_em.device))
        return z

    def combine(self, z, row_of, w, E: int):
        T, k = row_of.shape
        d = z.shape[1]
        y = torch.empty(T, d, dtype=torch.bfloat16, device=z.device)
        if T:
            B.moe_combine(z, row_of, w, y, B.MoEShape.of(T, d, E, k, 64))
        return y

    def ones(self, n: int, device):
        return torch.ones(n, 1, dtype=torch.float32, device=device)

    def check(self, ws) -> int:
        return B.moe_check(ws)


class TorchDistComm:
    """All-to-all exchanges over a ``torch.distributed`` process group (NCCL
    on GPUs, gloo on CPUs)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group

    def all_to_all(self, out: torch.Tensor, inp: torch.Tensor,
                   out_splits: Optional[List[int]] = None,
                   in_splits: Optional[List[int]] = None):
        self.dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)


class EPMoELayer:
    """One rank's share of an expert-parallel MoE layer: the full router
    (replicated), and the weights of its E/R local experts only."""

    def __init__(self, w_g: torch.Tensor, bias: Optional[torch.Tensor], w13_local: torch.Tensor,
                 w2_local: torch.Tensor, k: int, rank: int, world: int, ops=None, comm=None):
        self.w_g, self.bias = w_g, bias
        self.w13, self.w2 = w13_local, w2_local
        self.d, self.E = int(w_g.shape[0]), int(w_g.shape[1])
        self.k, self.rank, self.world = int(k), int(rank), int(world)
        self.E_loc = int(w13_local.shape[0])
        self.f = int(w2_local.shape[2])
        if self.E_loc * self.world != self.E:
            raise ValueError("every rank must hold E / world experts")
        self.ops = ops if ops is not None else LibraryOps()
        self.comm = comm

    # -------------------------------------------------------------- phases
    def dispatch_phase(self, x: torch.Tensor) -> dict:
        """Router, top-k and the rank-contiguous dispatch of this rank's tokens."""
        idx, w = self.ops.route(x, self.w_g, self.bias, self.k, self.f)
        st = self.ops.dispatch(idx, x, self.E, self.world, self.f)
        st.update(idx=idx, w=w, T=int(x.shape[0]))
        return st

    @staticmethod
    def split_rows(counts_host: torch.Tensor, world: int) -> List[int]:
        """Rows per destination (or source) rank from per-expert counts laid
        out [rank][local expert]."""
        return [int(v) for v in counts_host.view(world, -1).sum(dim=1).tolist()]

    def expert_phase(self, x_recv: torch.Tensor, recv_counts: torch.Tensor) -> dict:
        """The local experts over every row received, in received order."""
        N = int(x_recv.shape[0])
        eid = self.ops.recv_experts(recv_counts, self.world, self.E_loc, N)
        grp = self.ops.dispatch(eid.view(N, 1), x_recv, self.E_loc, 1, self.f)
        z_em = self.ops.ffn(grp["x_perm"], grp["offsets"], self.w13, self.w2, self.E_loc)
        z_recv = self.ops.combine(z_em, grp["row_of"], self.ops.ones(N, x_recv.device),
                                  self.E_loc)
        grp.update(expert_of_row=eid, z_em=z_em, z_recv=z_recv)
        return grp

    def combine_phase(self, st: dict, z_back: torch.Tensor) -> torch.Tensor:
        """The gate-weighted sum of each token's k returned rows."""
        return self.ops.combine(z_back, st["row_of"], st["w"], self.E)

    # -------------------------------------------------------------- one call
    def forward(self, x: torch.Tensor, keep: Optional[dict] = None) -> torch.Tensor:
        """The layer for this rank's tokens; every rank of the group calls it
        (the exchanges are collective).  ``keep`` (optional dict) receives the
        intermediate state for inspection."""
        if self.comm is None:
            raise RuntimeError("EPMoELayer.forward needs a communicator")
        st = self.dispatch_phase(x)
        counts = st["counts"]
        recv_counts = torch.empty_like(counts)
        self.comm.all_to_all(recv_counts, counts)  # E_loc counts per peer
        both = torch.cat([counts, recv_counts]).cpu()  # the one host synchronisation
        send_rows = self.split_rows(both[:self.E], self.world)
        recv_rows = self.split_rows(both[self.E:], self.world)
        x_recv = torch.empty(sum(recv_rows), self.d, dtype=x.dtype, device=x.device)
        self.comm.all_to_all(x_recv, st["x_perm"], recv_rows, send_rows)
        grp = self.expert_phase(x_recv, recv_counts)
        z_back = torch.empty(st["T"] * self.k, self.d, dtype=grp["z_recv"].dtype,
                             device=x.device)
        self.comm.all_to_all(z_back, grp["z_recv"], send_rows, recv_rows)
        y = self.combine_phase(st, z_back)
        if keep is not None:
            keep.update(st=st, grp=grp, send_rows=send_rows, recv_rows=recv_rows,
                        recv_counts=recv_counts, x_recv=x_recv, z_back=z_back)
        return y

    __call__ = forward

    def check(self, state: dict) -> int:
        """Device error word of a phase's workspace (synchronises)."""
        return self.ops.check(state["status"])
