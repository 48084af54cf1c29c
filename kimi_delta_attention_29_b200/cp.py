"""Context parallelism for one long sequence: the prefill split over the ranks of a process group.

Rank r holds a contiguous segment of the sequence's tokens.  The KDA recurrence is linear in the
pair (state, v) for fixed q, k, alpha and beta (Kimi Linear summary page, section "From linear
attention to Gated DeltaNet": S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
o_t = S_t^T q_t), so a segment acts on its incoming state as an affine map S_out = M S_in + b: b is
the segment's final state from a zero state and M = prod_t (I - beta_t k_t k_t^T) Diag(alpha_t) its
d_k x d_k transition, the final state of a pass with v = 0 from S_in = I.  One exchange step joins
the segments (section "Chunkwise parallel algorithm": each chunk's final state seeds the next; here
each segment's does): every rank all-gathers the [M | b] of all segments, the library composes them
into each segment's incoming state (kda_state_compose), and each rank runs its segment again from
that state for its outputs.  Per rank: one map pass of its segment (the intra-chunk work once, two
state passes per head: kda_segment_map), one all-gather of d_k (d_k + d_v) floats per head, the
composition (R small products per head) and one chunkwise prefill from the incoming state; rank 0
without h0 keeps the map pass's outputs.
"""
from __future__ import annotations

from typing import Callable, Sequence


def segment_map(q, k, v, log_alpha, beta, stream=None, workspace=None, want_o: bool = True):
    """One segment's outputs from a zero state (None unless want_o) and its map [M | b] [H, dk, dk + dv]
    (fp32).  q, k [1, T, H, dk], v [1, T, H, dv] with dv = dk; log_alpha [1, T, H, dk]; beta [1, T, H].
    On the tensor-core path (bf16, dk = dv = 128) one pass: kda_segment_map; otherwise two prefills, one
    from zero and one with v = 0 from the identity."""
    import torch
    from . import kda_chunk_fwd, kda_segment_map
    H, dk, dv = q.shape[2], q.shape[3], v.shape[3]
    if dk != dv:
        raise ValueError("the segment transition is formed as a state with dv = dk columns")
    if q.dtype == torch.bfloat16 and dk == 128:
        return kda_segment_map(q, k, v, log_alpha, beta, want_o=want_o, workspace=workspace, stream=stream)
    o0, b = kda_chunk_fwd(q, k, v, log_alpha, beta, None, None, workspace=workspace, stream=stream)
    eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(1, H, dk, dk).contiguous()
    _, M = kda_chunk_fwd(q, k, torch.zeros_like(v), log_alpha, beta, eye, None, workspace=workspace, stream=stream)
    return (o0 if want_o else None), torch.cat([M[0], b[0]], dim=2).contiguous()


def identity_map(H, dk, dv, device, dtype=None):
    """The map of an empty segment: [I | 0] (fp32 unless dtype is given)."""
    import torch
    dtype = dtype or torch.float32
    Mb = torch.zeros(H, dk, dk + dv, dtype=dtype, device=device)
    Mb[:, :, :dk] = torch.eye(dk, dtype=dtype, device=device)
    return Mb


def segment_from(q, k, v, log_alpha, beta, S_in, stream=None, workspace=None):
    """The segment's outputs from the incoming state S_in [H, dk, dv]."""
    from . import kda_chunk_fwd
    o, _ = kda_chunk_fwd(q, k, v, log_alpha, beta, S_in.unsqueeze(0).contiguous(), None, workspace=workspace,
                         stream=stream, output_final_state=False)
    return o


def kda_chunk_fwd_cp(q, k, v, log_alpha, beta, h0=None, group=None, stream=None, workspace=None,
                     segment: Callable | None = None, compose: Callable | None = None,
                     rerun: Callable | None = None, map_dtype=None):
    """Context-parallel prefill of one sequence over the ranks of `group` (torch.distributed; NCCL over
    NVLink on GPUs).  This rank's segment: q, k [1, T_r, H, dk], v [1, T_r, H, dv], log_alpha
    [1, T_r, H, dk], beta [1, T_r, H]; ranks hold consecutive segments in rank order (T_r may differ,
    0 included).  h0 [1, H, dk, dv] fp32 or None, the same on every rank.  Returns (o [1, T_r, H, dv],
    h_T [1, H, dk, dv]): this segment's outputs and the sequence's final state (on every rank).

    segment / compose / rerun default to segment_map, kda_state_compose and segment_from; tests on
    hosts without a GPU pass reference implementations of the same three steps.  Every rank sends its
    map in map_dtype (fp32 unless given; all ranks must agree)."""
    import torch
    import torch.distributed as dist
    from . import kda_state_compose
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    keep_o = rank == 0 and h0 is None  # the only rank whose map-pass outputs are final
    seg = segment or (lambda *a: segment_map(*a, stream=stream, workspace=workspace, want_o=keep_o))
    comp = compose or (lambda Mb, s0: kda_state_compose(Mb, s0, stream=stream))
    run = rerun or (lambda *a: segment_from(*a, stream=stream, workspace=workspace))
    map_dtype = map_dtype or torch.float32
    H, dk, dv = q.shape[2], q.shape[3], v.shape[3]
    o = None
    if q.shape[1] > 0:
        o, Mb = seg(q, k, v, log_alpha, beta)
        Mb = Mb.to(map_dtype)
    else:
        Mb = identity_map(H, dk, dv, q.device, map_dtype)
    parts = [torch.empty_like(Mb) for _ in range(world)]
    dist.all_gather(parts, Mb.contiguous(), group=group)  # the one exchange step
    gathered = torch.stack(parts).contiguous()
    S_in, S_out = comp(gathered, None if h0 is None else h0[0].contiguous())
    if q.shape[1] == 0:
        o = torch.empty_like(v)
    elif rank > 0 or h0 is not None:  # rank 0 without h0 already has its outputs
        o = run(q, k, v, log_alpha, beta, S_in[rank])
    return o, S_out.unsqueeze(0)


def kda_chunk_fwd_segments(q, k, v, log_alpha, beta, bounds: Sequence[int], h0=None, stream=None, workspace=None):
    """The same decomposition run segment by segment on one GPU without a process group: token ranges
    [bounds[j], bounds[j + 1]) play the ranks.  Returns (o, h_T) for the whole sequence."""
    import torch
    from . import kda_state_compose
    parts, outs, maps = [], [], []
    for a, e in zip(bounds[:-1], bounds[1:]):
        part = [x[:, a:e].contiguous() for x in (q, k, v, log_alpha, beta)]
        parts.append(part)
        if e > a:
            o0, Mb = segment_map(*part, stream=stream, workspace=workspace, want_o=(a == 0 and h0 is None))
        else:
            o0, Mb = torch.empty_like(part[2]), identity_map(q.shape[2], q.shape[3], v.shape[3], q.device)
        outs.append(o0)
        maps.append(Mb)
    S_in, S_out = kda_state_compose(torch.stack(maps).contiguous(), None if h0 is None else h0[0].contiguous(),
                                    stream=stream)
    for j, part in enumerate(parts):
        if part[0].shape[1] > 0 and (j > 0 or h0 is not None):
            outs[j] = segment_from(*part, S_in[j], stream=stream, workspace=workspace)
    return torch.cat(outs, dim=1), S_out.unsqueeze(0)
