"""Expert parallelism over a torch.distributed process group.

Each of the W ranks holds its own tokens and E / W of the experts: rank g holds
experts [g E/W, (g+1) E/W) and runs them on the rows routed to them from every rank.
The pages define a single-device layer; this split rests only on its structure: given
the routing, every expert's rows are independent of the others'.  One forward, on every
rank:

  1. route the rank's tokens (moe_route)                        -> idx, w [T, k]
  2. moe_permute: the routed rows in expert order, each row's expert as an index on
     the rank holding it, rows per expert, and the row of every slot (pos)
  3. rows for rank g = the rows of its experts (contiguous in expert order); the
     counts go to every rank (all-to-all of W integers)
  4. all-to-all of the rows, their experts and their routing weights
  5. moe_experts_forward on the rows received: this rank's experts
  6. all-to-all of the outputs back, with the splits of step 4 reversed
  7. moe_combine of the outputs in slot order (+ shared_output)        -> y

Every step on the data runs in the library's kernels (``LibraryOps``); this module
only sizes the exchange (one host copy of the E per-expert counts per forward, and one
of the W counts received) and calls the collectives.  With one rank the exchange is a
copy, nothing waits on the host, and the result equals moe_forward up to the order of
its fp32 sums.
"""
from __future__ import annotations

import types


# Tensors of the routing step, which the expert forward of routed rows does not take.
_ROUTER_INPUTS = ("router_weight", "router_logits", "logits", "router_bias", "selection_bias")


def _with(cfg, **kw):
    """A copy of a configuration object with some fields replaced."""
    d = dict(vars(cfg))
    d.update(kw)
    return types.SimpleNamespace(**d)


class LibraryOps:
    """The device steps, through the library's C ABI (device tensors on the current stream)."""

    def __init__(self):
        from . import (Workspace, _check, moe_combine, moe_experts_forward, moe_permute,
                       moe_workspace_size, options_of, route, shape_of, tensors_of)
        self._m = types.SimpleNamespace(Workspace=Workspace, check=_check, combine=moe_combine,
                                        experts_forward=moe_experts_forward, permute=moe_permute,
                                        workspace_size=moe_workspace_size, options_of=options_of,
                                        route=route, shape_of=shape_of, tensors_of=tensors_of)

    def _stream(self, t):
        import torch
        return torch.cuda.current_stream(t.device).cuda_stream

    def route(self, cfg, inputs):
        return self._m.route(cfg, inputs)

    def permute(self, cfg, idx, w, x, experts_per_rank):
        import torch
        m = self._m
        R = cfg.T * cfg.k
        shape, opts = m.shape_of(cfg), m.options_of(cfg)
        ws = m.Workspace(m.workspace_size(shape, opts), x.device)
        x_perm = torch.empty((R, cfg.d), dtype=x.dtype, device=x.device)
        row_expert = torch.empty(R, dtype=torch.int32, device=x.device)
        row_w = torch.empty(R, dtype=torch.float32, device=x.device)
        counts = torch.empty(cfg.E, dtype=torch.int32, device=x.device)
        pos = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=x.device)
        m.check(m.permute(shape, opts, idx.data_ptr(), w.data_ptr(), x.data_ptr(), x_perm.data_ptr(),
                          row_expert.data_ptr(), row_w.data_ptr(), counts.data_ptr(), pos.data_ptr(),
                          experts_per_rank, ws.ptr, ws.nbytes, self._stream(x)))
        return x_perm, row_expert, row_w, counts, pos

    def experts_forward(self, cfg_local, rows, row_expert, row_w, weights):
        import torch
        m = self._m
        y = torch.empty_like(rows)
        if rows.shape[0] == 0:
            return y
        shape, opts = m.shape_of(cfg_local), m.options_of(cfg_local)
        ws = m.Workspace(m.workspace_size(shape, opts), rows.device)
        experts = {k: v for k, v in weights.items() if k not in _ROUTER_INPUTS}  # rows come routed
        tens = m.tensors_of({**experts, "x": rows}, y)
        m.check(m.experts_forward(shape, opts, tens, row_expert.data_ptr(), row_w.data_ptr(), ws.ptr, ws.nbytes,
                                  self._stream(rows)))
        return y

    def combine(self, cfg, pos, Y, shared_output=None):
        import torch
        m = self._m
        y = torch.empty((cfg.T, cfg.d), dtype=Y.dtype, device=Y.device)
        so = 0 if shared_output is None else shared_output.data_ptr()
        m.check(m.combine(m.shape_of(cfg), pos.data_ptr(), Y.data_ptr(), Y.shape[0], so, y.data_ptr(),
                          self._stream(Y)))
        return y


class ExpertParallelMoE:
    """The MoE layer with its routed experts split over the ranks of ``group``.

    cfg: the layer's configuration (attributes as in moe_shape / moe_options; cfg.T is
    this rank's token count, cfg.E the total number of experts, Fs must be 0: a shared
    expert is computed by the caller and passed as shared_output).  local: this rank's
    expert tensors, gate_up / down (and their biases, gate / gate_bias for an unfused
    stack) of its E / W experts, plus router_bias / selection_bias for the routing and,
    to route on logits the layer computes (forward without logits), router_weight
    [d, E].
    """

    def __init__(self, cfg, local: dict, group=None, ops=None, host_exchange=None):
        """host_exchange: stage the exchanged tensors through host memory (for a backend
        without device collectives, such as gloo); default: when the group's backend is
        gloo."""
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        if cfg.E % self.world:
            raise ValueError(f"E={cfg.E} experts do not split over {self.world} ranks")
        if cfg.Fs:
            raise ValueError("a shared expert is not split: compute it apart and pass shared_output")
        self.cfg = cfg
        self.local = local
        self.ops = ops if ops is not None else LibraryOps()
        self.per_rank = cfg.E // self.world
        if host_exchange is None:
            host_exchange = self.world > 1 and dist.get_backend(group) == "gloo"
        self.host_exchange = host_exchange

    def _a2a(self, out, inp, out_splits, in_splits):
        if self.world == 1:
            out.copy_(inp)
        elif self.host_exchange and out.device.type != "cpu":
            o = out.new_empty(out.shape, device="cpu")
            self.dist.all_to_all_single(o, inp.to("cpu"), out_splits, in_splits, group=self.group)
            out.copy_(o)
        else:
            self.dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def forward(self, x, logits=None, shared_output=None):
        """y [T, d] for this rank's tokens x [T, d], routed on logits [T, E] or, when they
        are not given, on x . router_weight."""
        import torch
        cfg, ops, W, El = self.cfg, self.ops, self.world, self.per_rank
        T = x.shape[0]
        cfg_t = _with(cfg, T=T)
        inputs = {"x": x, "logits": logits, "router_bias": self.local.get("router_bias"),
                  "selection_bias": self.local.get("selection_bias")}
        if logits is None:
            if self.local.get("router_weight") is None:
                raise ValueError("forward needs logits, or router_weight in the rank's tensors")
            inputs["router_weight"] = self.local["router_weight"]
        idx, w = ops.route(cfg_t, inputs)
        x_perm, row_expert, row_w, counts, pos = ops.permute(cfg_t, idx, w, x, El if W > 1 else 0)
        if W == 1:  # every row stays: no split sizes to learn (and no host synchronisation)
            send = recv = [T * cfg.k]
        else:
            per_expert = counts.to("cpu").tolist()
            send = [sum(per_expert[g * El:(g + 1) * El]) for g in range(W)]
            send_t = torch.tensor(send, dtype=torch.int64, device=x.device)
            recv_t = torch.empty_like(send_t)
            self._a2a(recv_t, send_t, [1] * W, [1] * W)
            recv = recv_t.to("cpu").tolist()
        rows = sum(recv)
        x_recv = torch.empty((rows, cfg.d), dtype=x.dtype, device=x.device)
        e_recv = torch.empty(rows, dtype=torch.int32, device=x.device)
        w_recv = torch.empty(rows, dtype=torch.float32, device=x.device)
        self._a2a(x_recv, x_perm, recv, send)
        self._a2a(e_recv, row_expert, recv, send)
        self._a2a(w_recv, row_w, recv, send)
        cfg_local = _with(cfg, T=rows, E=El, k=1, Fs=0, shared_gate=False)
        y_recv = ops.experts_forward(cfg_local, x_recv, e_recv, w_recv, self.local)
        Y = torch.empty((x_perm.shape[0], cfg.d), dtype=y_recv.dtype, device=y_recv.device)
        self._a2a(Y, y_recv, send, recv)
        return ops.combine(cfg_t, pos, Y, shared_output)
