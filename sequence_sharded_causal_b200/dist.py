"""The D-GPU realisation: one process per GPU, each owning a contiguous range of the
logical zigzag shards.

"Folding Tensor and Sequence Parallelism" (summary page, section 2, attention layer)
gives every rank one zigzag shard of the sequence and rebuilds the full K/V context
with an all-gather before FlashAttention runs; the backward mirror image returns dK/dV
to the owning shards.  With N ranks and D logical shards (N divides D), rank q owns the
shards [q*D/N, (q+1)*D/N).  One training step of the attention core on rank q:

  1. all-gather K and V: every rank contributes its own rows, laid out shard-major
     ([D/N][B][2C][Hkv][d]); the gathered tensor is [D][B][2C][Hkv][d], which the
     kernels read directly (ZSA_KV_SHARD_MAJOR), so no reorder pass runs;
  2. zsa_attn_fwd restricted to the rank's shards: O and lse of its own rows;
  3. zsa_attn_bwd restricted to the rank's shards: dQ of its own rows and the partial
     dK / dV of the whole sequence from its own queries (shard-major layout);
  4. reduce-scatter dK and dV (sum): each rank receives its own rows, summed over every
     rank's queries.

This module is plumbing only: the collectives are torch.distributed calls (NCCL on
GPUs; the same calls run under gloo on CPU tensors in the tests), and every step of the
attention itself runs in libzsa's kernels.  Peer data reaches a rank's HBM through NCCL
before any kernel reads it; no kernel reads another GPU's memory.
"""
import torch

import sequence_sharded_causal_b200 as zsa


def shard_range(rank, world, D):
    """(shard_begin, shard_count) owned by `rank` of `world` ranks."""
    if world <= 0 or D % world != 0:
        raise ValueError(f"the {world} ranks must divide the D={D} logical shards")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    ns = D // world
    return rank * ns, ns


def gather_kv(k_local, v_local, group=None, out_k=None, out_v=None):
    """All-gather every rank's K / V rows ([ns][B][2C][Hkv][d] each) into the whole
    sequence in shard-major order ([D][B][2C][Hkv][d]), rank order = shard order."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    shape = (k_local.shape[0] * world,) + tuple(k_local.shape[1:])
    if out_k is None:
        out_k = torch.empty(shape, dtype=k_local.dtype, device=k_local.device)
    if out_v is None:
        out_v = torch.empty(shape, dtype=v_local.dtype, device=v_local.device)
    dist.all_gather_into_tensor(out_k, k_local.contiguous(), group=group)
    dist.all_gather_into_tensor(out_v, v_local.contiguous(), group=group)
    return out_k, out_v


def reduce_scatter_kv_grads(dk_part, dv_part, group=None, out_dk=None, out_dv=None):
    """Sum the ranks' partial dK / dV ([D][B][2C][Hkv][d], shard-major) and hand each
    rank its own rows ([ns][B][2C][Hkv][d])."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    shape = (dk_part.shape[0] // world,) + tuple(dk_part.shape[1:])
    if out_dk is None:
        out_dk = torch.empty(shape, dtype=dk_part.dtype, device=dk_part.device)
    if out_dv is None:
        out_dv = torch.empty(shape, dtype=dv_part.dtype, device=dv_part.device)
    dist.reduce_scatter_tensor(out_dk, dk_part.contiguous(), group=group)
    dist.reduce_scatter_tensor(out_dv, dv_part.contiguous(), group=group)
    return out_dk, out_dv


class ShardedAttention:
    """One rank's attention core of a D-shard zigzag run over an N-rank group.

    Holds the gathered K/V, the partial dK/dV and the workspaces, so that a step
    allocates nothing.  q / do / o / dq are the rank's own rows [ns][B][2C][Hq][d];
    k_local / v_local / dk / dv its own K/V rows [ns][B][2C][Hkv][d].
    """

    def __init__(self, B, S, Hq, Hkv, d, D, rank, world, group=None, causal=True, scale=None,
                 device=None):
        self.shard_begin, self.shard_count = shard_range(rank, world, D)
        self.group = group
        self.problem = zsa.make_problem(B, S, Hq, Hkv, d, D, causal, scale,
                                        kv_layout=zsa.ZSA_KV_SHARD_MAJOR,
                                        shard_begin=self.shard_begin,
                                        shard_count=self.shard_count)
        self.D, self.causal = D, causal
        twoC = S // D
        dev = device
        bf = torch.bfloat16
        self.k_all = torch.empty(D, B, twoC, Hkv, d, dtype=bf, device=dev)
        self.v_all = torch.empty_like(self.k_all)
        self.dk_part = torch.empty_like(self.k_all)
        self.dv_part = torch.empty_like(self.k_all)
        self.lse = torch.empty(self.shard_count, B, Hq, twoC, dtype=torch.float32, device=dev)
        self.ws_f = torch.empty(zsa.zsa_workspace_bytes(self.problem, 0), dtype=torch.uint8,
                                device=dev)
        self.ws_b = torch.empty(zsa.zsa_workspace_bytes(self.problem, 1), dtype=torch.uint8,
                                device=dev)

    def forward(self, q, k_local, v_local, o, stream=None):
        """Gather K/V, then O (into `o`) and lse of the rank's rows."""
        gather_kv(k_local, v_local, self.group, self.k_all, self.v_all)
        zsa.zsa_attn_fwd(self.problem, q, self.k_all, self.v_all, o, self.lse, self.ws_f,
                         stream=stream)
        return o, self.lse

    def backward(self, q, o, do, dq, dk, dv, stream=None):
        """dQ of the rank's rows (into `dq`) and its own rows of dK / dV (into `dk`, `dv`),
        summed over every rank's queries.  Uses the K/V gathered by forward()."""
        zsa.zsa_attn_bwd(self.problem, q, self.k_all, self.v_all, o, self.lse, do, dq,
                         self.dk_part, self.dv_part, self.ws_b, stream=stream)
        reduce_scatter_kv_grads(self.dk_part, self.dv_part, self.group, dk, dv)
        return dq, dk, dv

    def status(self):
        """Device status of both workspaces (synchronises): ZSA_OK or ZSA_ERR_TIMEOUT."""
        return zsa.zsa_device_status(self.ws_f) or zsa.zsa_device_status(self.ws_b)


# ---------------------------------------------------------------- TSP weight schedule
#
# "Folding Tensor and Sequence Parallelism" (summary page, section 2, attention layer):
# besides 1/D of the tokens, rank r holds one packed shard of the attention weights --
# the Q, K and V columns of its head group, and the rows of W_O for that group -- and the
# layer's projections iterate over the shards: at step s rank s broadcasts its shard and
# every rank projects its own tokens with it.  After the D steps each rank holds Q, K, V
# of all heads for its tokens (Q in the shard-major layout the attention kernels read,
# K / V as the rank's own rows for the all-gather), and the output projection's partials,
# one per step, summed.
#
# The broadcast of step s+1 is posted before the GEMM of step s is enqueued, so NCCL moves
# the next shard while the tensor cores work on the current one (double-buffered).

def qkv_columns(Hq, Hkv, d, D):
    """Columns of W_Q, W_K, W_V in each of the D packed shards: (nq, nk, nv)."""
    if (Hq * d) % D or (Hkv * d) % D:
        raise ValueError("the Q and K/V projection widths must split into D shards")
    return Hq * d // D, Hkv * d // D, Hkv * d // D


def pack_qkv_shard(wq, wk, wv, s, D):
    """Rank s's packed shard [hidden][nq + nk + nv] of W_Q [hidden][Hq*d], W_K, W_V."""
    nq, nk = wq.shape[1] // D, wk.shape[1] // D
    return torch.cat([wq[:, s * nq:(s + 1) * nq], wk[:, s * nk:(s + 1) * nk],
                      wv[:, s * nk:(s + 1) * nk]], dim=1).contiguous()


def wo_shard(wo, s, D):
    """Rank s's rows of W_O [Hq*d][hidden]: the inputs of its head group."""
    nq = wo.shape[0] // D
    return wo[s * nq:(s + 1) * nq].contiguous()


def _broadcast_steps(w_local, group, step_fn):
    """Run step_fn(s, w_s) for s = 0..world-1, W_s arriving by broadcast from rank s;
    the broadcast of s+1 overlaps step s."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    bufs = [torch.empty_like(w_local), torch.empty_like(w_local)]

    def post(s):
        b = w_local if s == rank else bufs[s % 2]
        src = dist.get_global_rank(group, s) if group is not None else s
        return b, dist.broadcast(b, src=src, group=group, async_op=True)

    cur = post(0)
    for s in range(world):
        nxt = post(s + 1) if s + 1 < world else None
        b, work = cur
        work.wait()
        step_fn(s, b)
        cur = nxt


def tsp_qkv_projection(x, w_local, q, k, v, Hq, Hkv, d, group=None, project=None,
                       status_ws=None, stream=None):
    """Q, K, V of the rank's tokens x [T][hidden] from the packed shards (this rank's is
    w_local [hidden][nq + nk + nv]).  q [T][Hq*d], k / v [T][Hkv*d] (bf16) are written."""
    import torch.distributed as dist
    D = dist.get_world_size(group)
    nq, nk, nv = qkv_columns(Hq, Hkv, d, D)
    if project is None:
        def project(s, w_s):
            zsa.zsa_tsp_project(x, w_s, [(q[:, s * nq:], Hq * d, nq, 0),
                                         (k[:, s * nk:], Hkv * d, nk, 0),
                                         (v[:, s * nv:], Hkv * d, nv, 0)], status_ws,
                                stream=stream)
    _broadcast_steps(w_local, group, project)
    return q, k, v


def tsp_out_projection(o, wo_local, y32, Hq, d, group=None, project=None, status_ws=None,
                       stream=None):
    """y32 [T][hidden] (fp32, zeroed here) = O W_O for the rank's tokens, o [T][Hq*d],
    summed over the steps' partials O[:, head group s] W_O[s] (this rank's rows:
    wo_local [nq][hidden])."""
    import torch.distributed as dist
    D = dist.get_world_size(group)
    nq = Hq * d // D
    y32.zero_()
    if project is None:
        def project(s, w_s):
            zsa.zsa_tsp_project(o[:, s * nq:], w_s, [(y32, y32.stride(0), y32.shape[1], 1)],
                                status_ws, T=o.shape[0], K=nq, N=y32.shape[1],
                                ldx=o.stride(0), stream=stream)
    _broadcast_steps(wo_local, group, project)
    return y32
