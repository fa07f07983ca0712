"""Head-sharded multi-GPU form of the path (the pages' standard setting: 8-way sequence parallelism,
fluxbbs.com "Hy-Nomas 拆解", sections 单卡 4090 怎么做到的 and 训练流程 (Ulysses, 2 of 16 heads per GPU);
hyphentech.top config table (8 GPUs, sp_size 8, full history)).

Activations arrive sequence-sharded: rank r holds tokens [r*S/G, (r+1)*S/G) of every head.  Attention,
its mask and the INT8 cache are independent per head, so each rank owns H/G heads: one all-to-all turns
its sequence shard of q / k / v into all tokens of its heads, the rank runs the library's append, mask
build and attention on its heads alone (its cache holds only them), and a second all-to-all returns
the output to the sequence layout.  Text K/V (at most 1280 tokens) are replicated and sliced by head.

The exchanges are torch.distributed all_to_all_single calls (NCCL between GPUs); every step of the
method itself runs in libnomas on the rank's own device memory.  No tensor of another GPU is handed to
a kernel.  Argument marshalling only, as the rest of the binding.
"""
from __future__ import annotations

import math
from typing import Optional

import torch
import torch.distributed as dist

from .runtime import KVCache


def _world(group) -> tuple:
    return dist.get_world_size(group), dist.get_rank(group)


def seq_to_heads(x: torch.Tensor, group=None) -> torch.Tensor:
    """[S/G, H, D] (this rank's tokens, every head) -> [S, H/G, D] (every token, this rank's heads).

    Tokens come out in global order (rank j's shard is tokens [j*S/G, (j+1)*S/G)); rank r gets heads
    [r*H/G, (r+1)*H/G)."""
    G, _ = _world(group)
    s_loc, H, D = x.shape
    if H % G:
        raise ValueError(f"{H} heads do not split over {G} ranks")
    send = x.reshape(s_loc, G, H // G, D).permute(1, 0, 2, 3).contiguous()   # [dest rank][token][head][D]
    recv = torch.empty_like(send)                                             # [source rank][token][head][D]
    dist.all_to_all_single(recv, send, group=group)
    return recv.reshape(G * s_loc, H // G, D)


def heads_to_seq(y: torch.Tensor, group=None) -> torch.Tensor:
    """[S, H/G, D] (every token, this rank's heads) -> [S/G, H, D] (this rank's tokens, every head)."""
    G, _ = _world(group)
    S, hg, D = y.shape
    if S % G:
        raise ValueError(f"{S} tokens do not split over {G} ranks")
    send = y.reshape(G, S // G, hg, D).contiguous()                           # [dest rank][token][head][D]
    recv = torch.empty_like(send)                                             # [source rank's heads][token]...
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3).reshape(S // G, G * hg, D)


def head_slice(x: Optional[torch.Tensor], rank: int, heads_per_rank: int) -> Optional[torch.Tensor]:
    """This rank's heads of a replicated [tokens, H, D] tensor, contiguous (every bf16 input of one
    library call shares one token stride)."""
    if x is None:
        return None
    return x[:, rank * heads_per_rank:(rank + 1) * heads_per_rank].contiguous()


class HeadShardedAttention:
    """The path on G ranks with H/G heads each (see the module docstring).  Sequence-sharded inputs and
    outputs; the rank's INT8 cache, masks and attention cover its own heads only."""

    def __init__(self, heads, head_dim, tokens_per_frame, window_frames, capacity_frames, head_store_tokens,
                 device, group=None):
        self.group = group
        self.G, self.rank = _world(group)
        if heads % self.G:
            raise ValueError(f"{heads} heads do not split over {self.G} ranks")
        self.H, self.hg, self.D = heads, heads // self.G, head_dim
        self.cache = KVCache(self.hg, head_dim, tokens_per_frame, window_frames, capacity_frames,
                             head_store_tokens, device)

    def append(self, k_loc, v_loc, n_frames, head_k=None, head_v=None, stream=None):
        """k_loc, v_loc: this rank's token shard [S/G, H, D] of the finished segment; head_k / head_v:
        the replicated description head [len, H, D] or None."""
        k = seq_to_heads(k_loc, self.group)
        v = seq_to_heads(v_loc, self.group)
        self.cache.append(k, v, n_frames, head_slice(head_k, self.rank, self.hg),
                          head_slice(head_v, self.rank, self.hg), stream=stream)

    def attention(self, seg, q_loc, k_loc, v_loc, ktxt, vtxt, mode=0, keep_frac=0.25, softmax_scale=None,
                  stream=None):
        """Returns fp32 [S/G, H, D]: this rank's tokens of the attention output, every head."""
        q = seq_to_heads(q_loc, self.group)
        k = seq_to_heads(k_loc, self.group)
        v = seq_to_heads(v_loc, self.group)
        kt = head_slice(ktxt, self.rank, self.hg)
        vt = head_slice(vtxt, self.rank, self.hg)
        buf, _ = self.cache.build_mask(seg, mode, keep_frac, q, k, stream=stream)
        scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(self.D)
        out, _ = self.cache.attention(seg, buf, q, k, v, kt, vt, scale, mode=mode, keep_frac=keep_frac,
                                      stream=stream)
        return heads_to_seq(out, self.group)
