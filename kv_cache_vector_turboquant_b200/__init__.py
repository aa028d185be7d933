"""TurboQuant KV-cache codec for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libtq.so`` behind the C ABI of
``include/tq.h``; this package is its ctypes binding plus a small convenience
layer with the call shapes of the "aither-kvcache" page ("Quick Start --
TurboQuant", "API Reference": ``TurboQuant(head_dim, bits, seed=42)``,
``encode(x) -> (packed, norms)``, ``decode(packed, norms)``,
``compression_ratio()``). PyTorch supplies device memory and streams only.
"""

from __future__ import annotations

from ._binding import (  # noqa: F401
    LIB_PATH,
    TQ_DEVERR_BLOCK_RANGE,
    TQ_DEVERR_POS_RANGE,
    TQ_DEVERR_SLOT_RANGE,
    TQ_DEVERR_SMEM_LAYOUT,
    TQ_DEVERR_TIMEOUT,
    TQ_ERR_ALIGNMENT,
    TQ_ERR_CUDA,
    TQ_ERR_DEVICE,
    TQ_ERR_INVALID_ARG,
    TQ_ERR_NOMEM,
    TQ_ERR_TIMEOUT,
    TQ_ERR_UNSUPPORTED,
    TQ_ERR_WORKSPACE,
    TQ_OK,
    TQ_PAGE_BLOCK,
    Ctx,
    TQError,
    TQ_ATTEND_STATIC_SCRATCH_BYTES,
    tq_attend_decode,
    tq_attend_decode_paged,
    tq_attend_decode_static,
    tq_attend_workspace_bytes,
    tq_create,
    tq_decode,
    tq_check_device_error,
    tq_device_error,
    tq_encode,
    tq_encode_append,
    tq_encode_append_kv,
    tq_encode_os,
    tq_decode_os,
    tq_encode_slots,
    tq_get_tables,
    tq_status_string,
    tq_tensor_core_check,
)


def _require(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


def _check(t, name: str, dtypes, shape=None, numel=None) -> None:
    """Type, dtype, layout and size of a tensor argument; the device is
    checked separately (_on_device), after every size check."""
    import torch

    _require(isinstance(t, torch.Tensor), f"{name}: a torch tensor")
    dtypes = dtypes if isinstance(dtypes, tuple) else (dtypes,)
    _require(t.dtype in dtypes, f"{name}: dtype {' or '.join(str(d) for d in dtypes)}, got {t.dtype}")
    _require(t.is_contiguous(), f"{name}: contiguous")
    if shape is not None:
        _require(tuple(t.shape) == tuple(shape), f"{name}: shape {tuple(shape)}, got {tuple(t.shape)}")
    if numel is not None:
        _require(t.numel() == numel, f"{name}: {numel} elements, got {t.numel()}")


def _on_device(**tensors) -> None:
    """Every kernel reads and writes device memory: host tensors are refused
    here, before a pointer reaches the library."""
    for name, t in tensors.items():
        _require(t.is_cuda, f"{name}: a CUDA tensor")


class TurboQuant:
    """One codec (head_dim, bits, seed) on the current CUDA device."""

    def __init__(self, head_dim: int = 128, bits: int = 4, seed: int = 42):
        self.ctx = tq_create(head_dim, bits, seed)
        self.head_dim, self.bits, self.seed = head_dim, bits, seed
        self.packed_bytes = self.ctx.packed_bytes

    def compression_ratio(self) -> float:
        """fp16 bytes over stored bytes (packed codes + f32 norm) per vector."""
        return 2.0 * self.head_dim / (self.packed_bytes + 4)

    def memory_report(self, seq_len: int, num_layers: int = 32, num_kv_heads: int = 8) -> dict:
        """KV-cache bytes of one sequence of `seq_len` tokens over `num_layers`
        layers of `num_kv_heads` kv heads (K and V), fp16 against this codec
        (packed codes plus one f32 norm per vector)."""
        vectors = 2 * int(num_layers) * int(num_kv_heads) * int(seq_len)
        fp16 = vectors * 2 * self.head_dim
        packed = vectors * (self.packed_bytes + 4)
        return {"vectors": vectors, "fp16_bytes": fp16, "packed_bytes": packed, "saved_bytes": fp16 - packed,
                "compression_ratio": fp16 / packed, "bits": self.bits, "head_dim": self.head_dim}

    def validate(self, num_vectors: int = 10000, seed: int = 0) -> dict:
        """Encode and decode `num_vectors` seeded N(0,1) fp16 vectors on the
        current device and report the reconstruction: mean relative squared
        error ||x - x_hat||^2 / ||x||^2, mean cosine similarity, and the
        largest relative error of the stored norms."""
        import torch

        g = torch.Generator(device="cuda").manual_seed(int(seed))
        x = torch.randn(int(num_vectors), self.head_dim, generator=g, device="cuda").to(torch.float16)
        packed, norms = self.encode(x)
        xh = self.decode(packed, norms).float()
        xf = x.float()
        nx = xf.norm(dim=1)
        rel = ((xf - xh).pow(2).sum(dim=1) / nx.pow(2)).mean().item()
        cos = torch.nn.functional.cosine_similarity(xf, xh, dim=1).mean().item()
        nerr = ((norms - xf.double().norm(dim=1).float()).abs() / nx).max().item()
        return {"num_vectors": int(num_vectors), "mse_relative": rel, "cosine": cos, "max_norm_rel_err": nerr,
                "bits": self.bits, "head_dim": self.head_dim}

    def benchmark(self, num_vectors: int = 32768, reps: int = 20) -> dict:
        """Device time of one encode and one decode of `num_vectors` vectors
        (CUDA events around `reps` back-to-back calls after a warm-up), with
        the fp16-equivalent throughput (2 * head_dim bytes per vector)."""
        import torch

        x = torch.randn(int(num_vectors), self.head_dim, device="cuda").to(torch.float16)
        packed, norms = self.encode(x)
        out = self.decode(packed, norms)
        res = {"num_vectors": int(num_vectors), "bits": self.bits, "head_dim": self.head_dim}
        for name, fn in (("encode", lambda: self.encode(x, out=(packed, norms))),
                         ("decode", lambda: self.decode(packed, norms, out=out))):
            for _ in range(3):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(int(reps)):
                fn()
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) / int(reps) / 1e3
            res[f"{name}_us"] = t * 1e6
            res[f"{name}_GBps"] = 2.0 * self.head_dim * int(num_vectors) / t / 1e9
        return res

    def encode(self, x, out=None, stream=None):
        """[..., d] fp16 CUDA tensor -> ([..., d*b/8] uint8, [...] float32)."""
        import torch

        _require(x.is_cuda and x.dtype == torch.float16 and x.is_contiguous(), "x: contiguous fp16 CUDA tensor")
        _require(x.shape[-1] == self.head_dim, "last dim must be head_dim")
        lead = tuple(x.shape[:-1])
        n = x.numel() // self.head_dim
        if out is None:
            packed = torch.empty(lead + (self.packed_bytes,), dtype=torch.uint8, device=x.device)
            norms = torch.empty(lead, dtype=torch.float32, device=x.device)
        else:
            packed, norms = out
            _check(packed, "out packed", torch.uint8, numel=n * self.packed_bytes)
            _check(norms, "out norms", torch.float32, numel=n)
            _on_device(packed=packed, norms=norms)
        tq_encode(self.ctx, x, n, packed, norms, stream)
        return packed, norms

    def decode(self, packed, norms, out=None, stream=None):
        """([..., d*b/8] uint8, [...] float32) -> [..., d] fp16."""
        import torch

        _require(packed.is_cuda and packed.dtype == torch.uint8 and packed.is_contiguous(), "packed: uint8 CUDA")
        _require(packed.shape[-1] == self.packed_bytes, "last dim of packed must be head_dim*bits/8")
        _require(norms.dtype == torch.float32 and norms.is_contiguous(), "norms: contiguous float32")
        lead = tuple(packed.shape[:-1])
        n = packed.numel() // self.packed_bytes
        _require(norms.numel() == n, "norms must have one entry per vector")
        x = out if out is not None else torch.empty(lead + (self.head_dim,), dtype=torch.float16,
                                                    device=packed.device)
        _check(x, "out", torch.float16, numel=n * self.head_dim)
        _on_device(norms=norms, out=x)
        tq_decode(self.ctx, packed, norms, n, x, stream)
        return x

    def encode_append(self, x, cache_packed, cache_norms, slot, stream=None):
        """Write one token per sequence: x [n_seq, h, d] into cache slot[s]."""
        import torch

        _require(x.dim() == 3 and x.shape[-1] == self.head_dim, "x: [n_seq, h, head_dim]")
        n_seq, h, d = x.shape
        _require(cache_packed.dim() == 4, "cache_packed: [n_seq, s_max, h, P]")
        s_max = cache_packed.shape[1]
        _check(x, "x", torch.float16)
        _check(cache_packed, "cache_packed", torch.uint8, shape=(n_seq, s_max, h, self.packed_bytes))
        _check(cache_norms, "cache_norms", torch.float32, shape=(n_seq, s_max, h))
        _check(slot, "slot", torch.int32, numel=n_seq)
        _on_device(x=x, cache_packed=cache_packed, cache_norms=cache_norms, slot=slot)
        tq_encode_append(self.ctx, x, n_seq, h, cache_packed, cache_norms, s_max, slot, stream)

    def encode_append_kv(self, k, v, k_cache, k_norms, v_cache, v_norms, slot, stream=None):
        """Write the key and the value of one token per sequence in one launch:
        k, v [n_seq, h, d] into slot[s] of their caches [n_seq, s_max, h, P]."""
        import torch

        _require(k.dim() == 3 and k.shape[-1] == self.head_dim and tuple(v.shape) == tuple(k.shape),
                 "k, v: [n_seq, h, head_dim]")
        n_seq, h, d = k.shape
        _require(k_cache.dim() == 4, "k_cache: [n_seq, s_max, h, P]")
        s_max = k_cache.shape[1]
        for name, t in (("k", k), ("v", v)):
            _check(t, name, torch.float16)
        for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
            _check(t, name, torch.uint8, shape=(n_seq, s_max, h, self.packed_bytes))
        for name, t in (("k_norms", k_norms), ("v_norms", v_norms)):
            _check(t, name, torch.float32, shape=(n_seq, s_max, h))
        _check(slot, "slot", torch.int32, numel=n_seq)
        _on_device(k=k, v=v, k_cache=k_cache, v_cache=v_cache, k_norms=k_norms, v_norms=v_norms, slot=slot)
        tq_encode_append_kv(self.ctx, k, v, n_seq, h, k_cache, k_norms, v_cache, v_norms, s_max, slot, stream)

    def encode_os(self, x, stream=None):
        """Offset + fp16-scale variant: x [..., d] fp16 -> (packed [..., P]
        uint8, side [...] int32 = fp16 offset | fp16 scale << 16)."""
        import torch

        _require(x.shape[-1] == self.head_dim, "last dim must be head_dim")
        _check(x, "x", torch.float16)
        _on_device(x=x)
        lead = x.shape[:-1]
        n = x.numel() // self.head_dim
        packed = torch.empty(*lead, self.packed_bytes, dtype=torch.uint8, device=x.device)
        side = torch.empty(lead, dtype=torch.int32, device=x.device)
        tq_encode_os(self.ctx, x, n, packed, side, stream)
        return packed, side

    def decode_os(self, packed, side, stream=None):
        import torch

        _require(packed.shape[-1] == self.packed_bytes, "last dim of packed must be head_dim*bits/8")
        lead = packed.shape[:-1]
        n = packed.numel() // self.packed_bytes
        _check(packed, "packed", torch.uint8)
        _check(side, "side", (torch.int32, torch.uint32), numel=n)
        _on_device(packed=packed, side=side)
        out = torch.empty(*lead, self.head_dim, dtype=torch.float16, device=packed.device)
        tq_decode_os(self.ctx, packed, side, n, out, stream)
        return out

    def encode_slots(self, x, cache_packed, cache_norms, slot_mapping, stream=None):
        """Encode-on-write: x [n_tok, h, d] into slot slot_mapping[t] of a pool
        cache_packed [num_slots, h, P] (or a paged pool [num_blocks, 16, h, P]),
        cache_norms likewise; negative slots are skipped."""
        import torch

        _require(x.dim() == 3 and x.shape[-1] == self.head_dim, "x: [n_tok, h, head_dim]")
        n_tok, h, d = x.shape
        _require(cache_packed.shape[-2] == h and cache_packed.shape[-1] == self.packed_bytes, "cache layout")
        num_slots = cache_packed.numel() // (h * self.packed_bytes)
        _check(x, "x", torch.float16)
        _check(cache_packed, "cache_packed", torch.uint8)
        _check(cache_norms, "cache_norms", torch.float32, numel=num_slots * h)
        _check(slot_mapping, "slot_mapping", torch.int32, numel=n_tok)
        _on_device(x=x, cache_packed=cache_packed, cache_norms=cache_norms, slot_mapping=slot_mapping)
        tq_encode_slots(self.ctx, x, n_tok, h, cache_packed, cache_norms, num_slots, slot_mapping, stream)


def attend_decode(q, k_codec: TurboQuant, v_codec: TurboQuant, k_packed, k_norms, v_packed, v_norms,
                  positions, out=None, workspace=None, stream=None):
    """One decode step of attention over packed caches.

    q [B, Hq, d] fp16; k_packed [B, S, Hkv, Pk] uint8; k_norms [B, S, Hkv] f32;
    v likewise; positions [B] int32 (valid cache length per sequence).
    Returns o [B, Hq, d] fp16.
    """
    import torch

    _require(q.dim() == 3 and k_packed.dim() == 4, "q: [B, Hq, d]; k_packed: [B, S, Hkv, Pk]")
    B, hq, d = q.shape
    s_max, hkv = k_packed.shape[1], k_packed.shape[2]
    _check(q, "q", torch.float16)
    _check(k_packed, "k_packed", torch.uint8, shape=(B, s_max, hkv, k_codec.packed_bytes))
    _check(v_packed, "v_packed", torch.uint8, shape=(B, s_max, hkv, v_codec.packed_bytes))
    _check(k_norms, "k_norms", torch.float32, shape=(B, s_max, hkv))
    _check(v_norms, "v_norms", torch.float32, shape=(B, s_max, hkv))
    _check(positions, "positions", torch.int32, numel=B)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", torch.float16, shape=(B, hq, d))
    ws_bytes = tq_attend_workspace_bytes(B, hq, d, s_max)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    _check(workspace, "workspace", torch.uint8)
    _on_device(q=q, k_packed=k_packed, v_packed=v_packed, k_norms=k_norms, v_norms=v_norms, positions=positions,
               out=out, workspace=workspace)
    tq_attend_decode(k_codec.ctx, v_codec.ctx, q, B, hq, hkv, k_packed, k_norms, v_packed, v_norms, s_max,
                     positions, out, workspace, workspace.numel(), stream)
    return out


class TQPagedAttention:
    """Decode-step attention over paged packed caches, in the form of the
    pages' `TQPagedAttention(tq, num_query_heads).forward(...)`: `tq` codes
    the keys and, unless `v_tq` is given, the values too."""

    def __init__(self, tq: TurboQuant, num_query_heads: int, v_tq: TurboQuant = None):
        self.k_codec, self.v_codec = tq, (v_tq if v_tq is not None else tq)
        self.num_query_heads = int(num_query_heads)

    def forward(self, query, k_packed, k_norms, v_packed, v_norms, block_tables, context_lens, out=None,
                workspace=None, stream=None):
        """query [B, num_query_heads, head_dim] fp16; caches [num_blocks, 16,
        Hkv, P]; block_tables [B, max_blocks] int32; context_lens [B] int32.
        Returns [B, num_query_heads, head_dim] fp16."""
        _require(query.dim() == 3 and query.shape[1] == self.num_query_heads,
                 "query must be [B, num_query_heads, head_dim]")
        return attend_decode_paged(query, self.k_codec, self.v_codec, k_packed, k_norms, v_packed, v_norms,
                                   block_tables, context_lens, out=out, workspace=workspace, stream=stream)

    __call__ = forward


def attend_decode_paged(q, k_codec: TurboQuant, v_codec: TurboQuant, k_cache, k_norms, v_cache, v_norms,
                        block_tables, context_lens, out=None, workspace=None, stream=None):
    """One decode step of attention over paged packed caches.

    q [B, Hq, d] fp16; k_cache [num_blocks, 16, Hkv, Pk] uint8; k_norms
    [num_blocks, 16, Hkv] f32; v likewise; block_tables [B, max_blocks] int32
    (block of positions [16 j, 16 j + 16) of sequence b); context_lens [B]
    int32. Returns o [B, Hq, d] fp16.
    """
    import torch

    _require(q.dim() == 3 and k_cache.dim() == 4 and block_tables.dim() == 2,
             "q: [B, Hq, d]; k_cache: [num_blocks, 16, Hkv, Pk]; block_tables: [B, max_blocks]")
    B, hq, d = q.shape
    num_blocks, blk, hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    _require(blk == TQ_PAGE_BLOCK, f"cache blocks must hold {TQ_PAGE_BLOCK} positions")
    max_blocks = block_tables.shape[1]
    _check(q, "q", torch.float16)
    _check(k_cache, "k_cache", torch.uint8, shape=(num_blocks, blk, hkv, k_codec.packed_bytes))
    _check(v_cache, "v_cache", torch.uint8, shape=(num_blocks, blk, hkv, v_codec.packed_bytes))
    _check(k_norms, "k_norms", torch.float32, shape=(num_blocks, blk, hkv))
    _check(v_norms, "v_norms", torch.float32, shape=(num_blocks, blk, hkv))
    _check(block_tables, "block_tables", torch.int32, shape=(B, max_blocks))
    _check(context_lens, "context_lens", torch.int32, numel=B)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", torch.float16, shape=(B, hq, d))
    ws_bytes = tq_attend_workspace_bytes(B, hq, d, max_blocks * TQ_PAGE_BLOCK)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    _check(workspace, "workspace", torch.uint8)
    _on_device(q=q, k_cache=k_cache, v_cache=v_cache, k_norms=k_norms, v_norms=v_norms, block_tables=block_tables,
               context_lens=context_lens, out=out, workspace=workspace)
    tq_attend_decode_paged(k_codec.ctx, v_codec.ctx, q, B, hq, hkv, k_cache, k_norms, v_cache, v_norms, num_blocks,
                           block_tables, max_blocks, context_lens, out, workspace, workspace.numel(), stream)
    return out
