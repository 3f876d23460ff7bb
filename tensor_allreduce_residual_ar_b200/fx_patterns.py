"""Graph rewrites that route the unfused "all-reduce, residual add, RMSNorm"
subgraphs of a traced torch program to the fused operators
``torch.ops.ar_b200.*`` (the library's kernels).

The PR #50802 report ("实现拆解" item 1, "关键源码片段") describes pattern
replacements for the two-output form (normalised output and the new
residual), the output-only form whose residual result is dead, the site with
no residual (all_reduce -> rms_norm), and the per-group FP8 quantisation of
the normalised output with the 16-bit output kept for a second consumer;
the PR #54787 report adds the Gemma weighting (weight bias 1.0).  Here the
all-reduce of the tensor-parallel ranks' partials is, on one GPU, their sum:
a chain of additions of W >= 2 partial tensors.

Recognised (in torch.fx graphs from ``symbolic_trace`` or aten-level
graphs):

    s  = all_reduce_sum_reference([p0, ..., p_{W-1}])   # or p0 + p1 + ... + p_{W-1}
    r  = s + residual                        # optional (no-residual site)
    y  = rms_norm(r, (H,), weight, eps)      # or rms_norm(r, (H,), None, eps) * (1 + w)
    q, scales = quant_fp8_group_reference(y) # optional, per-group FP8

and the tensor-parallel form of the same sites, where each rank holds one
partial and the all-reduce crosses GPUs (the pages' own setting):

    s  = tp_all_reduce_reference(p, comm)    # comm: a ``comm.register`` id
    ...                                      # then as above

which is rewritten to ``torch.ops.ar_b200.tp_*`` (the all-reduce pulled
over the communicator inside the fused kernel).  The marker is matched as
the one node ``symbolic_trace`` keeps for it; torch's functional collectives
in an aten-level graph are not matched.

``fuse_allreduce_rmsnorm(gm)`` rewrites every match in place and returns the
count per form.  Reading of the pages where they are silent: for
``a + b`` feeding the norm, a side that is itself an addition used only there
is the partial sum and the other side the residual; an addition of two plain
tensors is the no-residual sum of two partials (the result is the same sum
either way; only the kernel's summation order differs).
"""
from __future__ import annotations

import operator

import torch
import torch.fx as fx
import torch.nn.functional as F

from . import torch_ops  # noqa: F401  (registers torch.ops.ar_b200.*)


def quant_fp8_group_reference(y: torch.Tensor, group: int = 128):
    """The unfused per-group FP8 quantisation the rewrite recognises after a
    norm: per group of `group` elements along the last dimension,
    scale = amax / 448 and codes = e4m3fn(y / scale) (saturating), returned
    as (codes [..., H] float8_e4m3fn, scales [..., H / group] fp32).  A
    traced graph keeps it as one node (``torch.fx.wrap``)."""
    g = y.float().unflatten(-1, (-1, group))
    scale = g.abs().amax(-1, keepdim=True) / 448.0
    q = (g / scale).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).flatten(-2)
    return q, scale.squeeze(-1)


def all_reduce_sum_reference(partials):
    """The all-reduce of W partials that sit on one device, as the unfused
    program writes it: their elementwise sum (left to right, in the inputs'
    dtype).  A traced graph keeps it as one node, which marks the partial
    sum unambiguously (a plain chain of additions is recognised too)."""
    out = partials[0]
    for p in partials[1:]:
        out = out + p
    return out


def tp_all_reduce_reference(x: torch.Tensor, comm: int) -> torch.Tensor:
    """The tensor-parallel all-reduce (sum) of this rank's partial over the
    ranks of the communicator registered as `comm`, as the unfused program
    writes it: a copy, all-reduced through torch.distributed over the
    communicator's process group (at world size 1, the copy).  A traced
    graph keeps it as one node."""
    from . import comm as C
    c = C.lookup(comm)
    out = x.clone()
    if c.world > 1:
        import torch.distributed as dist
        dist.all_reduce(out, group=c.group)
    return out


torch.fx.wrap("quant_fp8_group_reference")
torch.fx.wrap("all_reduce_sum_reference")
torch.fx.wrap("tp_all_reduce_reference")

_ADDS = {operator.add, torch.add, torch.ops.aten.add.Tensor}
_NORMS = {F.rms_norm, torch.rms_norm, torch.ops.aten.rms_norm.default}
_MULS = {operator.mul, torch.mul, torch.ops.aten.mul.Tensor}
_SHAPE_USES = {"size", "shape", "dim", "dtype", "device"}


def _is_add(n) -> bool:
    return isinstance(n, fx.Node) and n.op == "call_function" and n.target in _ADDS and \
        len(n.args) == 2 and not n.kwargs.get("alpha")


def _is_meta_use(u: fx.Node) -> bool:
    """A use that reads only metadata (shape, dtype, ...), not the data."""
    if u.op == "call_function" and u.target is getattr and u.args[1] in _SHAPE_USES:
        return True
    return u.op == "call_method" and u.target in ("size", "dim")


def _data_users(n: fx.Node):
    return [u for u in n.users if not _is_meta_use(u)]


def _is_zero(a) -> bool:
    return isinstance(a, (int, float)) and a == 0


def _leaves(n, root: bool = True):
    """Operands of an addition tree whose inner additions are used only
    inside the tree; a constant zero (from Python's sum) is dropped."""
    if _is_add(n) and (root or len(_data_users(n)) == 1):
        out = []
        for a in n.args:
            if _is_zero(a):
                continue
            sub = _leaves(a, root=False)
            if sub is None:
                return None
            out += sub
        return out
    if isinstance(n, fx.Node):
        return [n]
    return None            # a non-zero constant term: not a sum of tensors


def _norm_parts(n: fx.Node):
    """(x, weight, eps, gemma, the node whose result is y, nodes computing
    the Gemma weight 1 + w) for an RMSNorm node, or None."""
    if n.op != "call_function" or n.target not in _NORMS:
        return None
    args = list(n.args) + [None] * 4
    x = args[0]
    weight = n.kwargs.get("weight", args[2])
    eps = n.kwargs.get("eps", args[3])
    if eps is None or not isinstance(eps, (int, float)):
        return None
    if weight is not None:
        return x, weight, float(eps), False, n, []
    # Gemma: rms_norm without weight, times (1 + w)
    users = _data_users(n)
    if len(users) != 1:
        return None
    m = users[0]
    if m.op != "call_function" or m.target not in _MULS or len(m.args) != 2:
        return None
    other = m.args[1] if m.args[0] is n else m.args[0]
    if not _is_add(other):
        return None
    a, b = other.args
    w = b if isinstance(a, (int, float)) and a == 1 else a if isinstance(b, (int, float)) and b == 1 else None
    if not isinstance(w, fx.Node):
        return None
    return x, w, float(eps), True, m, [other]


def _is_marked_sum(n) -> bool:
    return isinstance(n, fx.Node) and n.op == "call_function" and n.target is all_reduce_sum_reference \
        and len(n.args) == 1 and isinstance(n.args[0], (list, tuple)) and len(n.args[0]) >= 1 \
        and all(isinstance(a, fx.Node) for a in n.args[0])


def _is_tp_sum(n) -> bool:
    return isinstance(n, fx.Node) and n.op == "call_function" and n.target is tp_all_reduce_reference \
        and len(n.args) == 2 and isinstance(n.args[0], fx.Node) and isinstance(n.args[1], int) \
        and not n.kwargs


def _split_sum(x: fx.Node):
    """(partials, residual or None, communicator id or None) for the norm's
    input, or None."""
    if _is_marked_sum(x):
        return list(x.args[0]), None, None
    if _is_tp_sum(x):
        return [x.args[0]], None, x.args[1]
    if not _is_add(x):
        return None
    a, b = x.args
    for s, res in ((a, b), (b, a)):
        if _is_tp_sum(s) and len(_data_users(s)) == 1 and isinstance(res, fx.Node):
            return [s.args[0]], res, s.args[1]
    for s, res in ((a, b), (b, a)):
        if _is_marked_sum(s) and len(_data_users(s)) == 1 and isinstance(res, fx.Node):
            return list(s.args[0]), res, None
    for s, res in ((a, b), (b, a)):
        if _is_add(s) and len(_data_users(s)) == 1 and isinstance(res, fx.Node):
            parts = _leaves(s)
            if parts and len(parts) >= 2:
                return parts, res, None
    parts = _leaves(x)
    if parts and len(parts) >= 2:
        return parts, None, None
    return None


def _erase_dead(graph: fx.Graph, nodes):
    """Erase the given nodes that no longer have users, following their
    operands among them (the replaced subgraph only; nothing else of the
    program is touched)."""
    pending = [n for n in nodes if isinstance(n, fx.Node)]
    changed = True
    while changed:
        changed = False
        for n in list(pending):
            if n.graph is graph and not n.users:
                graph.erase_node(n)
                pending.remove(n)
                changed = True


def fuse_allreduce_rmsnorm(gm: fx.GraphModule) -> dict:
    """Rewrite every recognised subgraph of ``gm`` to the fused operators.
    Returns the number of rewrites per form: "two_output", "out_only",
    "no_residual" (counted in addition to the first two), "fp8", "gemma",
    and "tp" (the tensor-parallel ones among them)."""
    graph = gm.graph
    counts = {"two_output": 0, "out_only": 0, "no_residual": 0, "fp8": 0, "gemma": 0, "tp": 0}
    for node in list(graph.nodes):
        if node.graph is not graph:
            continue
        np_ = _norm_parts(node)
        if np_ is None:
            continue
        x, weight, eps, gemma, y_node, extra = np_
        split = _split_sum(x) if isinstance(x, fx.Node) else None
        if split is None:
            continue
        parts, residual, comm = split
        tp = comm is not None
        # the fused operators' leading arguments: the W partials, or this
        # rank's partial; the communicator id goes last
        lead = parts[0] if tp else list(parts)
        tail = (comm,) if tp else ()
        # the residual result (r = x) is live if anything other than the
        # norm reads its data
        r_live = any(u is not node for u in _data_users(x))
        y_users = _data_users(y_node)
        quant = [u for u in y_users if u.op == "call_function" and u.target is quant_fp8_group_reference
                 and len(u.args) >= 1 and u.args[0] is y_node
                 and (len(u.args) < 2 or u.args[1] == 128) and u.kwargs.get("group", 128) == 128]
        # the fused call goes right after the last of its operands (the sum,
        # the residual, the weight); every reader of r must come after it
        order = {n: i for i, n in enumerate(graph.nodes)}
        anchor = max([x] + [a for a in (residual, weight) if isinstance(a, fx.Node)],
                     key=lambda n: order[n])
        if any(order[u] <= order[anchor] for u in _data_users(x) if u is not node):
            continue
        with graph.inserting_before(anchor.next):
            if quant:
                op = torch.ops.ar_b200.tp_add_rmsnorm_fp8_group if tp else torch.ops.ar_b200.add_rmsnorm_fp8_group
                fused = graph.call_function(op.default, (lead, residual, weight, eps, gemma) + tail)
                q_ = graph.call_function(operator.getitem, (fused, 0))
                s_ = graph.call_function(operator.getitem, (fused, 1))
                y_ = graph.call_function(operator.getitem, (fused, 2))
                r_ = graph.call_function(operator.getitem, (fused, 3))
                qn = quant[0]
                for u in list(qn.users):
                    if u.op == "call_function" and u.target is operator.getitem and u.args[1] in (0, 1):
                        u.replace_all_uses_with(q_ if u.args[1] == 0 else s_)
                graph_nodes_to_drop = [u for u in list(qn.users)] + [qn]
                y_node.replace_all_uses_with(y_)
                counts["fp8"] += 1
            elif r_live:
                op = torch.ops.ar_b200.tp_add_rmsnorm if tp else torch.ops.ar_b200.add_rmsnorm
                fused = graph.call_function(op.default, (lead, residual, weight, eps, gemma) + tail)
                y_ = graph.call_function(operator.getitem, (fused, 0))
                r_ = graph.call_function(operator.getitem, (fused, 1))
                y_node.replace_all_uses_with(y_)
                graph_nodes_to_drop = []
                counts["two_output"] += 1
            else:
                op = torch.ops.ar_b200.tp_add_rmsnorm_out_only if tp else torch.ops.ar_b200.add_rmsnorm_out_only
                y_ = graph.call_function(op.default, (lead, residual, weight, eps, gemma) + tail)
                r_ = None
                y_node.replace_all_uses_with(y_)
                graph_nodes_to_drop = []
                counts["out_only"] += 1
        if r_ is not None:
            x.replace_all_uses_with(r_, delete_user_cb=lambda u: u is not node)
        else:
            # only metadata reads of r remain: read them from the first partial
            for u in list(x.users):
                if u is not node and _is_meta_use(u):
                    u.replace_input_with(x, parts[0])
        counts["no_residual"] += residual is None
        counts["gemma"] += gemma
        counts["tp"] += tp
        sum_tree, stack = [], [x]
        while stack:
            n = stack.pop()
            if (_is_add(n) or _is_marked_sum(n) or _is_tp_sum(n)) and n not in parts:
                sum_tree.append(n)
                stack += [a for a in n.all_input_nodes]
        # the norm's shape argument (getattr / getitem / size of r)
        shape_nodes, stack = [], list(node.all_input_nodes)
        while stack:
            n = stack.pop()
            if n.op in ("call_function", "call_method") and (_is_meta_use(n) or n.target is operator.getitem) \
                    and n not in parts and n is not residual and n is not weight:
                shape_nodes.append(n)
                stack += list(n.all_input_nodes)
        cand = []
        for n in graph_nodes_to_drop + [y_node, node] + extra + shape_nodes + sum_tree:
            if n not in cand:
                cand.append(n)
        _erase_dead(graph, cand)
    graph.lint()
    gm.recompile()
    return counts
