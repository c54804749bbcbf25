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
