"""One denoising step on the token stream, driven through the C ABI.

The block stack runs on the CFG pair (the same x and timestep against the
conditional and the unconditional context, batched as B = 2), then
wan_euler_cfg_step combines the two outputs with the guidance scale and
moves x by (sigma_next - sigma) * v ("Wan2.2 code walkthrough" (newtid.com),
sampling-loop snippet). Device memory comes from torch; every step of the
computation runs in libwan.
"""
from __future__ import annotations

import torch

from . import synth, wan
from .configs import BlockConfig


class DenoiseStep:
    def __init__(self, cfg: BlockConfig, seed: int = 0, device: str = "cuda", weights=None,
                 fp8: bool = False, attn8: bool = False):
        """``fp8``: the blocks run their projections as FP8 GEMMs (the bf16
        weights are quantized per tensor once, here); ``attn8`` also runs the
        self-attention as the 8-bit attention."""
        self.cfg = cfg
        self.dims = wan.dims_of(cfg)
        self.device = device
        self.weights = weights if weights is not None else synth.step_weights(cfg, device, seed)
        if fp8 or attn8:
            self.dims.dtype = wan.WAN_FP8_ATTN if attn8 else wan.WAN_FP8
            self.weights = [wan.quantize_block_weights(w) for w in self.weights]
        self.cweights = [wan.make_weights(w) for w in self.weights]
        acts = synth.block_activations(2, cfg.L, cfg.dim, cfg.text_len, cfg.dtype, device,
                                       seed + 100, same_e0=True)
        self.x = acts["x"][0].contiguous()                 # [L, D] float32, the state
        self.ctx = acts["ctx"]                             # [2, T, D]: cond, uncond
        self.e0 = acts["e0"]                               # [2, 6, D], one timestep
        self.xb = torch.empty((2, cfg.L, cfg.dim), dtype=torch.float32, device=device)
        self.rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta, device=device)
        self.ws = wan.alloc_workspace(self.dims, 2, device=device)
        self.ws_bytes = self.ws.numel()

    def blocks(self, stream=None):
        """The block stack on xb (in place)."""
        s = wan._stream(stream)
        for cw in self.cweights:
            wan.check(wan.wan_block_forward(self.dims, 2, self.xb.data_ptr(), self.ctx.data_ptr(),
                                            None, self.e0.data_ptr(), cw, self.rope.data_ptr(),
                                            self.rope.shape[0], self.ws.data_ptr(), self.ws_bytes,
                                            s))

    def step(self, stream=None):
        c = self.cfg
        self.xb[0].copy_(self.x)
        self.xb[1].copy_(self.x)
        self.blocks(stream)
        wan.check(wan.wan_euler_cfg_step(self.x.data_ptr(), self.xb[0].data_ptr(),
                                         self.xb[1].data_ptr(), wan.WAN_F32, self.x.numel(),
                                         c.guide_scale, c.sigma, c.sigma_next,
                                         wan._stream(stream)))
        return self.x



def cfg_pairs(world: int):
    """Rank pairs of the CFG-parallel step: ranks 2p and 2p + 1 run the
    conditional and the unconditional branch of one denoising step."""
    if world < 2 or world % 2:
        raise ValueError(f"the CFG-parallel step needs an even number of ranks, got {world}")
    return [[2 * p, 2 * p + 1] for p in range(world // 2)]


def cfg_exchange(local, gathered, group):
    """All-gather of the pair's two block outputs: ``local`` is this rank's
    [1, L, D] output, ``gathered`` [2, L, D] receives the conditional one
    (the pair's first rank) at 0 and the unconditional one at 1. NCCL writes
    straight into ``gathered`` (over NVLink between GPUs of one node); other
    backends gather into its two rows."""
    import torch.distributed as dist
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(gathered, local, group=group)
    else:
        dist.all_gather([gathered[0], gathered[1]], local[0], group=group)


class CFGParallelStep:
    """The denoising step of DenoiseStep with the CFG pair split over two
    ranks (two GPUs): each rank runs the block stack on its branch alone
    (B = 1, its own context, the shared x and timestep), the two block
    outputs are exchanged within the pair, and each rank applies
    wan_euler_cfg_step to its own copy of x, so both copies stay equal. With
    the same seed the inputs and weights are those of DenoiseStep, and since
    no kernel mixes sequences, each rank's branch output equals that
    sequence of the batched step.

    ``branch`` 0 = conditional, 1 = unconditional (the rank's index within
    ``group``, a process group of the two ranks)."""

    def __init__(self, cfg: BlockConfig, branch: int, group, seed: int = 0, device: str = "cuda",
                 weights=None):
        if branch not in (0, 1):
            raise ValueError(f"branch must be 0 (conditional) or 1 (unconditional), got {branch}")
        self.cfg = cfg
        self.branch = branch
        self.group = group
        self.dims = wan.dims_of(cfg)
        self.device = device
        self.weights = weights if weights is not None else synth.step_weights(cfg, device, seed)
        self.cweights = [wan.make_weights(w) for w in self.weights]
        acts = synth.block_activations(2, cfg.L, cfg.dim, cfg.text_len, cfg.dtype, device,
                                       seed + 100, same_e0=True)
        self.x = acts["x"][0].contiguous()                              # [L, D] float32, the state
        self.ctx = acts["ctx"][branch:branch + 1].contiguous()          # [1, T, D]: this branch
        self.e0 = acts["e0"][branch:branch + 1].contiguous()            # [1, 6, D]
        self.xb = torch.empty((1, cfg.L, cfg.dim), dtype=torch.float32, device=device)
        self.v = torch.empty((2, cfg.L, cfg.dim), dtype=torch.float32, device=device)
        self.rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta, device=device)
        self.ws = wan.alloc_workspace(self.dims, 1, device=device)
        self.ws_bytes = self.ws.numel()

    def blocks(self, stream=None):
        """This branch's block stack on xb (in place)."""
        s = wan._stream(stream)
        for cw in self.cweights:
            wan.check(wan.wan_block_forward(self.dims, 1, self.xb.data_ptr(), self.ctx.data_ptr(),
                                            None, self.e0.data_ptr(), cw, self.rope.data_ptr(),
                                            self.rope.shape[0], self.ws.data_ptr(), self.ws_bytes,
                                            s))

    def step(self, stream=None):
        """One step; the copy, the blocks, the exchange and the update are
        ordered on ``stream`` (a torch CUDA stream; default the current one)."""
        c = self.cfg
        stream = stream if stream is not None else torch.cuda.current_stream()
        with torch.cuda.stream(stream):
            self.xb[0].copy_(self.x)
            self.blocks(stream)
            cfg_exchange(self.xb, self.v, self.group)
            wan.check(wan.wan_euler_cfg_step(self.x.data_ptr(), self.v[0].data_ptr(), self.v[1].data_ptr(),
                                             wan.WAN_F32, self.x.numel(), c.guide_scale, c.sigma,
                                             c.sigma_next, wan._stream(stream)))
        return self.x

def permute_chunks_device(src, dst, dims, perm, chunk_bytes, stream=None):
    """dst = src with its chunk axes permuted, by wan_permute_chunks."""
    wan.check(wan.wan_permute_chunks(src.data_ptr(), dst.data_ptr(), len(dims), dims, perm, chunk_bytes,
                                     wan._stream(stream)))


def seq_head_exchange(send, recv, group):
    """The all-to-all of the head-parallel attention: ``send`` and ``recv``
    are [N, ...] with block j of ``send`` going to rank j of ``group`` and
    block i of ``recv`` coming from rank i. NCCL moves device buffers
    directly (over NVLink between GPUs of one node); other backends stage
    through host memory."""
    import torch.distributed as dist
    if dist.get_backend(group) == "nccl":
        dist.all_to_all_single(recv, send, group=group)
    else:
        r = torch.empty(recv.shape, dtype=recv.dtype)
        dist.all_to_all_single(r, send.cpu(), group=group)
        recv.copy_(r)


class UlyssesExchange:
    """Buffers and layout changes of the head-parallel (Ulysses) attention
    for one of N ranks ("Wan paper deep dive" (charles2530.github.io),
    training/inference-system section: Ulysses inside Ring). Rank r holds
    tokens [r rows, (r + 1) rows) of each of B sequences and, between the
    two all-to-alls, heads [r hl, (r + 1) hl) of all L = N rows tokens
    (hl = heads / N). Layouts (chunks of hl * d elements):

      q|k|v rows  [B][rows][3][N][hl d]    (wan_block_sp_qkv output)
      send_qkv    [N][B][rows][3][hl d]    block j -> rank j
      recv_qkv    [N][B][rows][3][hl d]    block i <- rank i (tokens of shard i)
      qkv_heads   [3][B][N rows][hl d]     dense q, k, v of this rank's heads
      o_heads     [B][N rows][hl d]        attention output, this rank's heads
      send_o      [N][B][rows][hl d]       tokens of shard j -> rank j
      recv_o      [N][B][rows][hl d]       heads of rank i
      o_rows      [B][rows][N][hl d]       all heads of this rank's rows

    ``permute`` and ``exchange`` default to wan_permute_chunks and
    seq_head_exchange; tests pass host versions."""

    def __init__(self, B, L, N, heads, head_dim, dtype, group=None, device="cuda", permute=None,
                 exchange=None):
        if N < 1 or L % N or heads % N:
            raise ValueError(f"{N} ranks must divide the {L} tokens and the {heads} heads")
        self.B, self.L, self.N, self.rows, self.hl, self.d = B, L, N, L // N, heads // N, head_dim
        self.group = group
        self.permute = permute or permute_chunks_device
        self.exchange = exchange or seq_head_exchange
        c = self.hl * head_dim
        self.chunk_elems = c
        self.chunk_bytes = c * torch.empty((), dtype=dtype).element_size()
        B, rows = self.B, self.rows
        mk = lambda *shape: torch.empty(shape, dtype=dtype, device=device)
        self.qkv_rows = mk(B, rows, 3 * N * c)
        self.send_qkv = mk(N, B, rows, 3, c)
        self.recv_qkv = mk(N, B, rows, 3, c)
        self.qkv_heads = mk(3, B, N * rows, c)
        self.o_heads = mk(B, N * rows, c)
        self.send_o = mk(N, B, rows, c)
        self.recv_o = mk(N, B, rows, c)
        self.o_rows = mk(B, rows, N * c)

    def pack_qkv(self, stream=None):
        self.permute(self.qkv_rows, self.send_qkv, (self.B, self.rows, 3, self.N), (3, 0, 1, 2),
                     self.chunk_bytes, stream)

    def unpack_qkv(self, stream=None):
        self.permute(self.recv_qkv, self.qkv_heads, (self.N, self.B, self.rows, 3), (3, 1, 0, 2),
                     self.chunk_bytes, stream)

    def pack_o(self, stream=None):
        self.permute(self.o_heads, self.send_o, (self.B, self.N, self.rows), (1, 0, 2), self.chunk_bytes, stream)

    def unpack_o(self, stream=None):
        self.permute(self.recv_o, self.o_rows, (self.N, self.B, self.rows), (1, 2, 0), self.chunk_bytes, stream)

    def to_heads(self, stream=None):
        """qkv_rows (this rank's tokens, all heads) -> qkv_heads (all tokens,
        this rank's heads)."""
        self.pack_qkv(stream)
        self.exchange(self.send_qkv, self.recv_qkv, self.group)
        self.unpack_qkv(stream)

    def to_rows(self, stream=None):
        """o_heads (all tokens, this rank's heads) -> o_rows (this rank's
        tokens, all heads)."""
        self.pack_o(stream)
        self.exchange(self.send_o, self.recv_o, self.group)
        self.unpack_o(stream)


class UlyssesStep:
    """The denoising step of DenoiseStep with every block's self-attention
    head-parallel over the N ranks of ``group``: rank r keeps tokens
    [r L/N, (r + 1) L/N) of x (and of the CFG pair's block inputs), runs
    wan_block_sp_qkv on them, exchanges q, k, v so that it holds all tokens
    of heads [r n/N, (r + 1) n/N), runs wan_attention on those, exchanges the
    outputs back and runs wan_block_sp_finish on its tokens. The CFG-Euler
    update is elementwise, so each rank moves its own tokens. With the same
    seed the inputs and weights are those of DenoiseStep; no kernel mixes
    tokens of different shards except the attention, which sees whole
    sequences, so the union of the ranks' x equals the single-rank phase
    path (N = 1) bit for bit."""

    def __init__(self, cfg: BlockConfig, rank: int, N: int, group=None, seed: int = 0, device: str = "cuda",
                 weights=None, exchange=None):
        if cfg.L % N or cfg.heads % N:
            raise ValueError(f"{N} ranks must divide L = {cfg.L} and heads = {cfg.heads}")
        self.cfg, self.rank, self.N = cfg, rank, N
        self.rows = cfg.L // N
        self.tok0 = rank * self.rows
        self.dims = wan.dims_of(cfg)
        self.weights = weights if weights is not None else synth.step_weights(cfg, device, seed)
        self.cweights = [wan.make_weights(w) for w in self.weights]
        acts = synth.block_activations(2, cfg.L, cfg.dim, cfg.text_len, cfg.dtype, device, seed + 100,
                                       same_e0=True)
        self.x = acts["x"][0, self.tok0:self.tok0 + self.rows].contiguous()   # [rows, D], this shard
        self.ctx = acts["ctx"]
        self.e0 = acts["e0"]
        del acts
        self.xb = torch.empty((2, self.rows, cfg.dim), dtype=torch.float32, device=device)
        self.rope = wan.rope_freqs(cfg.head_dim, 1024, cfg.theta, device=device)
        n = wan.wan_block_sp_workspace_bytes(self.dims, 2, self.rows)
        if n == 0:
            raise wan.WanError(wan.WAN_EINVAL, wan.last_error())
        self.ws = torch.empty(n, dtype=torch.uint8, device=device)
        self.ex = UlyssesExchange(2, cfg.L, N, cfg.heads, cfg.head_dim, synth.TORCH_DTYPES[cfg.dtype], group,
                                  device, exchange=exchange)
        self.hl = cfg.heads // N

    def block_qkv(self, i, stream=None):
        wan.check(wan.wan_block_sp_qkv(self.dims, 2, self.rows, self.tok0, self.xb.data_ptr(), self.e0.data_ptr(),
                                       self.cweights[i], self.rope.data_ptr(), self.rope.shape[0],
                                       self.ex.qkv_rows.data_ptr(), self.ws.data_ptr(), self.ws.numel(),
                                       wan._stream(stream)))

    def block_attention(self, stream=None):
        q, k, v = self.ex.qkv_heads[0], self.ex.qkv_heads[1], self.ex.qkv_heads[2]
        c = self.cfg
        wan.check(wan.wan_attention(2, self.hl, c.L, c.L, c.head_dim, self.dims.dtype, q.data_ptr(), k.data_ptr(),
                                    v.data_ptr(), self.ex.o_heads.data_ptr(), None, 0.0, None, None, 0,
                                    wan._stream(stream)))

    def block_finish(self, i, stream=None):
        wan.check(wan.wan_block_sp_finish(self.dims, 2, self.rows, self.xb.data_ptr(), self.ctx.data_ptr(), None,
                                          self.e0.data_ptr(), self.cweights[i], self.ex.o_rows.data_ptr(),
                                          self.ws.data_ptr(), self.ws.numel(), wan._stream(stream)))

    def euler(self, stream=None):
        c = self.cfg
        wan.check(wan.wan_euler_cfg_step(self.x.data_ptr(), self.xb[0].data_ptr(), self.xb[1].data_ptr(),
                                         wan.WAN_F32, self.x.numel(), c.guide_scale, c.sigma, c.sigma_next,
                                         wan._stream(stream)))

    def step(self, stream=None):
        self.xb[0].copy_(self.x)
        self.xb[1].copy_(self.x)
        for i in range(len(self.cweights)):
            self.block_qkv(i, stream)
            self.ex.to_heads(stream)
            self.block_attention(stream)
            self.ex.to_rows(stream)
            self.block_finish(i, stream)
        self.euler(stream)
        return self.x


class ModelDenoiseStep:
    """One CFG flow-matching Euler step on the latent through the whole model
    (wan_model_forward on the CFG pair at t = 1000 sigma, then
    wan_euler_cfg_step on the latent). With two experts, the high-noise one
    runs while t >= boundary ("Wan2.2 code walkthrough" (newtid.com), MoE
    snippet: boundary 0.875 * 1000 for text-to-video, 900 for image-to-video).

    ``experts`` maps "high" / "low" to (model weight dict, list of block weight
    dicts); a single expert may be passed as {"high": ...} with boundary 0.
    """

    def __init__(self, dims: "wan.wan_model_dims", experts: dict, text, latent,
                 boundary: float = 875.0, ctx_lens=None, rope_max_pos: int = 1024,
                 theta: float = 1e4, device: str = "cuda"):
        self.dims = dims
        self.boundary = boundary
        self.experts = {k: (wan.make_model_weights(mw), wan.make_block_array(bl))
                        for k, (mw, bl) in experts.items()}
        self._keep = experts                         # device tensors stay alive
        self.text = text                             # [2, T, text_dim]: cond, uncond
        self.ctx_lens = ctx_lens
        self.latent = latent                         # [C_in, F, H, W] float32, the state
        head_dim = dims.dim // dims.heads
        self.rope = wan.rope_freqs(head_dim, rope_max_pos, theta, device=device)
        self.lat2 = torch.empty((2,) + tuple(latent.shape), dtype=torch.float32, device=device)
        self.t = torch.empty(2, dtype=torch.float32, device=device)
        self.v = torch.empty((2, dims.C_out, dims.F, dims.H, dims.W), dtype=torch.float32,
                             device=device)
        self.ws = wan.alloc_model_workspace(dims, 2, device=device)

    def expert(self, sigma: float) -> str:
        t = 1000.0 * sigma
        if "low" not in self.experts or t >= self.boundary:
            return "high"
        return "low"

    def _guide(self, name, guide_scale):
        """A (low-noise, high-noise) pair picks the expert's scale ([WALK]
        sampling-loop snippet: e.g. (3.0, 4.0) for text-to-video)."""
        if isinstance(guide_scale, (tuple, list)):
            return guide_scale[1] if name == "high" else guide_scale[0]
        return guide_scale

    def velocity(self, sigma: float, stream=None):
        """The model on the CFG pair at t = 1000 sigma: self.v[0] (cond),
        self.v[1] (uncond). Returns the expert used."""
        s = wan._stream(stream)
        name = self.expert(sigma)
        mw, blocks = self.experts[name]
        self.lat2[0].copy_(self.latent)
        self.lat2[1].copy_(self.latent)
        self.t.fill_(1000.0 * sigma)
        wan.check(wan.wan_model_forward(self.dims, 2, self.lat2.data_ptr(), self.t.data_ptr(),
                                        wan._ptr(self.text), wan._ptr(self.ctx_lens), mw, blocks,
                                        len(blocks), self.rope.data_ptr(), self.rope.shape[0],
                                        self.v.data_ptr(), self.ws.data_ptr(), self.ws.numel(), s))
        return name

    def step(self, sigma: float, sigma_next: float, guide_scale, stream=None):
        """Euler step from sigma to sigma_next."""
        name = self.velocity(sigma, stream)
        wan.check(wan.wan_euler_cfg_step(self.latent.data_ptr(), self.v[0].data_ptr(),
                                         self.v[1].data_ptr(), wan.WAN_F32, self.latent.numel(),
                                         self._guide(name, guide_scale), sigma, sigma_next,
                                         wan._stream(stream)))
        return self.latent

    def unipc_step(self, sampler: "wan.UniPCSampler", guide_scale, stream=None):
        """One UniPC step (the sampler's x is this latent): the model at the
        sampler's current sigma, then the fused UniPC update."""
        name = self.velocity(sampler.sigma, stream)
        sampler.step(self.v[0], self.v[1], self._guide(name, guide_scale), stream)
        return self.latent
