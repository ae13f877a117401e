"""The tree-MTP verification forward step of a 27B-class dense model, composed
from the library's C-ABI calls (nothing here computes; every op is a kernel).

Per layer (pre-norm decoder block, 16 tree nodes = 16 rows):
    RMSNorm + NVFP4 quantise -> QKV linear -> FP8 KV append of the 16 nodes
    -> tree attention over the paged FP8 cache -> quantise -> O linear
    (+ residual, in place) -> RMSNorm + quantise -> gate+up linear
    -> SwiGLU + quantise -> down linear (+ residual, in place).
After the last layer: RMSNorm + quantise -> LM head -> per-node argmax.
Before the layers, kv_page_restore copies the reused prompt prefix (96% of
the context) from the prefix cache into the live pool ("KV-cache reuse
between agent steps"); the 16-node tree is verified in one forward pass
("Tree multi-token prediction"); weights, activations and the LM head are
NVFP4 and the cache is FP8 ("NVFP4 and FP8").

Suffix prefill (VerifyModel.prefill) writes the K/V of the prompt tokens that
the prefix cache does not hold ("KV-cache reuse between agent steps": only the
new suffix is prefilled) with the many-token kernels: every glue op over all S
rows in one launch, the NVFP4 linears as tiles of 128 weight rows x 256 tokens
(nvfp4_linear_wide), and causal attention in blocks of 128 queries, block b
attending to everything before it plus its own causal chain.

All buffers are allocated once, so a step can be captured in a CUDA graph.
"""
from __future__ import annotations

import contextlib
import math

import numpy as np
import torch

from . import inputs as I
from . import lib as nv

PAGE_BYTES = I.N_KV_HEADS * I.PAGE * I.HEAD_DIM      # one (layer, K|V, page) plane: 32 KB
PREFILL_CHUNK = 128                                  # queries per causal-attention launch
PREFILL_STREAMS = 8                                  # streams the blocks of a layer's attention share
PREFILL_ATTN_SPLITS = 3                              # context splits per query head of a block while >= 4 overlap


def prefill_chunks(start: int, S: int, C: int = PREFILL_CHUNK):
    """Query blocks of a suffix prefill's attention: (row0, rows, ctx_len) for
    rows row0 .. row0+rows-1 of the S suffix tokens, which sit at positions
    start+row0 ..; ctx_len = start+row0 is the context each block attends to
    in full before its own causal chain."""
    if start < 0 or S < 0 or C < 1:
        raise ValueError("need start >= 0, S >= 0, C >= 1")
    return [(r, min(C, S - r), start + r) for r in range(0, S, C)]


class Linear:
    """NVFP4 weight in the linear kernel's tile image (codes + scales) and its
    fp32 tensor scale g."""

    def __init__(self, prep, g, N, K):
        self.prep, self.g, self.N, self.K = prep, g, N, K

    @property
    def nbytes(self):
        """Algorithmic weight bytes (codes + E4M3 block scales)."""
        return self.N * self.K // 2 + self.N * self.K // 16

    @staticmethod
    def from_fp32(w: torch.Tensor):
        N, K = w.shape
        codes, scales, g = nv.quantize(w)
        prep = nv.prepare_weight(codes, scales, N, K)
        del codes, scales
        return Linear(prep, g, N, K)


class Act:
    """A quantised activation: prepared tile image + tensor scale."""

    def __init__(self, K, dev):
        self.K = K
        self.buf = nv.act_buffer(K, dev)
        self.g = torch.empty(1, dtype=torch.float32, device=dev)

    @property
    def out(self):
        return (None, None, self.g)


class VerifyModel:
    """64-layer NVFP4 model + paged FP8 KV cache + prefix cache, on one GPU.

    weights="device": N(0, 0.02) weights drawn on the GPU (torch generator,
    seeded per layer) -- same distribution as the host generator, used for
    timing; weights="host": the seeded numpy generator of `inputs` (layer l,
    tensor t -> inputs.weight_fp32(4, t, N, K, sub=l)), which the oracle
    reproduces.

    first_layer: the model holds layers first_layer .. first_layer+n_layers-1
    of the stack (their weights; the cache and the scales are the slice's
    own), e.g. one layer deep in the 64-layer stack for a per-layer check."""

    SITES = 4      # quantisation sites per layer: norm1, attention out, norm2, SwiGLU

    def __init__(self, n_layers=I.N_LAYERS, ctx_len=I.CTX_MAX, T=I.TREE_NODES, weights="device",
                 prefix_frac=0.96, device="cuda", lm_head=True, seed=42, first_layer=0):
        self.dev = torch.device(device)
        # activation tensor scales: dynamic (amax/2688 per call) until calibrate()
        # turns them into static per-site scales, as a calibrated checkpoint has
        self.static = False
        self._record = False
        self.n_layers, self.L, self.T = n_layers, ctx_len, T
        self.eps = 1e-6
        H, F, Hq, Hkv, D, P = I.HIDDEN, I.FFN, I.N_Q_HEADS, I.N_KV_HEADS, I.HEAD_DIM, I.PAGE
        self.layers = []
        gen = torch.Generator(device=self.dev)
        for l in range(first_layer, first_layer + n_layers):
            lay = {}
            for t, (name, (K, N)) in enumerate(I.LAYER_LINEARS.items()):
                if weights == "host":
                    w = torch.from_numpy(I.weight_fp32(4, t, N, K, sub=l)).to(self.dev)
                else:
                    gen.manual_seed(seed * 1000003 + l * 17 + t)
                    w = torch.randn(N, K, generator=gen, device=self.dev, dtype=torch.float32).mul_(I.W_STD)
                lay[name] = Linear.from_fp32(w)
                del w
            self.layers.append(lay)
        self.norm_w = torch.ones(2 * n_layers + 1, H, dtype=torch.bfloat16, device=self.dev)
        self.lm_head = None
        if lm_head:
            if weights == "host":
                w = torch.from_numpy(I.weight_fp32(4, 9, I.VOCAB, H)).to(self.dev)
            else:
                gen.manual_seed(seed * 1000003 + 999)
                w = torch.randn(I.VOCAB, H, generator=gen, device=self.dev).mul_(I.W_STD)
            self.lm_head = Linear.from_fp32(w)
            del w
        torch.cuda.empty_cache()

        self.prefix_frac, self._cache_seed = prefix_frac, seed + first_layer
        self.set_context(ctx_len)

        # activations (static buffers)
        self.h = torch.empty(T, H, dtype=torch.bfloat16, device=self.dev)
        self.parent = torch.empty(T, dtype=torch.int32, device=self.dev)
        self.qkv = torch.empty(T, (Hq + 2 * Hkv) * D, dtype=torch.bfloat16, device=self.dev)
        self.attn = torch.empty(T, Hq * D, dtype=torch.bfloat16, device=self.dev)
        self.gu = torch.empty(T, 2 * F, dtype=torch.bfloat16, device=self.dev)
        self.q_h = Act(H, self.dev)
        self.q_a = Act(Hq * D, self.dev)
        self.q_f = Act(F, self.dev)
        self.logits = torch.empty(T, I.VOCAB, dtype=torch.bfloat16, device=self.dev)
        self.ids = torch.empty(T, dtype=torch.int32, device=self.dev)
        self.G = torch.ones(n_layers * self.SITES + 1, dtype=torch.float32, device=self.dev)

    def set_context(self, ctx_len):
        """(Re)build the paged FP8 cache for ctx_len cached tokens, keeping the
        weights: planes (layer, K|V) x pool pages x 32 KB in a randomly
        permuted pool, the prefix cache holding round(prefix_frac * ctx_len)
        tokens, and the restore ids.  CUDA graphs captured before hold the old
        buffers and must be captured again."""
        P, T, n_layers = I.PAGE, self.T, self.n_layers
        self.kv = self.src = None
        if self.dev.type == "cuda":
            torch.cuda.empty_cache()
        self.L = ctx_len
        self.n_log = math.ceil((ctx_len + T) / P)
        self.n_pool = self.n_log + 8
        g = I.rng(4, 500)
        self.page_table_h = g.permutation(self.n_pool)[:self.n_log].astype(np.int32)
        self.page_table = torch.from_numpy(self.page_table_h).to(self.dev)
        # prefix cache (hot cache of the previous agent turn) and restore ids
        self.prefix_tokens = int(round(self.prefix_frac * ctx_len))
        self.n_prefix_pages = math.ceil(self.prefix_tokens / P)
        self.n_src = self.n_prefix_pages + 16
        self.kv = torch.empty(n_layers, 2, self.n_pool, PAGE_BYTES, dtype=torch.uint8, device=self.dev)
        self.src = torch.empty(n_layers, 2, self.n_src, PAGE_BYTES, dtype=torch.uint8, device=self.dev)
        self.k_scale = torch.empty(n_layers, I.N_KV_HEADS, dtype=torch.float32, device=self.dev)
        self.v_scale = torch.empty(n_layers, I.N_KV_HEADS, dtype=torch.float32, device=self.dev)
        self._fill_cache(self._cache_seed)
        src_pages = g.permutation(self.n_src)[:self.n_prefix_pages]
        planes = np.arange(n_layers * 2)[:, None]
        self.src_ids = torch.from_numpy((planes * self.n_src + src_pages[None, :]).ravel().astype(np.int32)).to(self.dev)
        self.dst_ids = torch.from_numpy(
            (planes * self.n_pool + self.page_table_h[None, :self.n_prefix_pages]).ravel().astype(np.int32)).to(self.dev)

    def _fill_cache(self, seed):
        """Cache contents as in the single-layer attention workload: K and V
        ~ N(0,1), stored as FP8 E4M3 with one scale per (layer, KV head, K|V)
        = amax/448 over that head's live and prefix-cache planes (so the
        restored pages and the live ones share a scale), cast with torch's
        float8_e4m3fn conversion.  Drawn on the GPU (torch generator)."""
        Hkv = I.N_KV_HEADS
        gen = torch.Generator(device=self.dev)
        gen.manual_seed(int(np.random.default_rng([42, 4, 501, seed]).integers(1 << 62)))
        for l in range(self.n_layers):
            for kv, scale in ((0, self.k_scale), (1, self.v_scale)):
                live = torch.randn(self.n_pool, Hkv, PAGE_BYTES // Hkv, generator=gen, device=self.dev)
                pre = torch.randn(self.n_src, Hkv, PAGE_BYTES // Hkv, generator=gen, device=self.dev)
                amax = torch.maximum(live.abs().amax(dim=(0, 2)), pre.abs().amax(dim=(0, 2)))
                sc = amax / 448.0
                scale[l].copy_(sc)
                for buf, x in ((self.kv, live), (self.src, pre)):
                    buf[l, kv].view(-1, Hkv, PAGE_BYTES // Hkv).copy_(
                        (x / sc[None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8))
                del live, pre

    # ------------------------------------------------------------------ pools
    def k_pool(self, l):
        return self.kv[l, 0].view(self.n_pool, I.N_KV_HEADS, I.PAGE, I.HEAD_DIM)

    def v_pool(self, l):
        return self.kv[l, 1].view(self.n_pool, I.N_KV_HEADS, I.HEAD_DIM * I.PAGE)

    # ------------------------------------------------------------------ ops
    def restore(self):
        nv.kv_page_restore(self.src.view(-1), self.src_ids, self.kv.view(-1), self.dst_ids, PAGE_BYTES)

    # ------------------------------------------------------------------ scales
    def _site(self, i):
        """Static scale of quantisation site i (device [1]), or None when dynamic."""
        return self.G[i:i + 1] if self.static else None

    def _note(self, i, act):
        if self._record:
            self.G[i:i + 1].copy_(act.g)

    def calibrate(self, restore=True):
        """Run one step with dynamic tensor scales and keep each site's scale as
        its static g_in from then on (one activation scale per quantised tensor
        of the checkpoint)."""
        self.static, self._record = False, True
        self.step(restore=restore)
        self._record, self.static = False, True

    def layer(self, l):
        lay, T = self.layers[l], self.T
        s0 = l * self.SITES
        nv.rmsnorm_quantize(self.h, self.norm_w[2 * l], self.eps, self.q_h.out, act=self.q_h.buf,
                            g_in=self._site(s0))
        self._note(s0, self.q_h)
        self._linear(self.q_h.buf, self.q_h.g, lay["qkv"], self.qkv)
        qd = I.N_Q_HEADS * I.HEAD_DIM
        kd = I.N_KV_HEADS * I.HEAD_DIM
        nv.kv_append(self.qkv[:, qd:], self.qkv[:, qd + kd:], self.qkv.stride(0), T, self.k_pool(l),
                     self.v_pool(l), self.page_table, self.L, self.k_scale[l], self.v_scale[l])
        if self.static:
            # attention output quantised in the combine launch with the static scale
            g_a = self._site(s0 + 1)
            nv.tree_attn(self.qkv, self.k_pool(l), self.v_pool(l), self.page_table, self.L, self.parent,
                         self.k_scale[l], self.v_scale[l], out=self.attn, ld_q=self.qkv.stride(0), T=T,
                         Hq=I.N_Q_HEADS, g_act=g_a, act=self.q_a.buf)
        else:
            nv.tree_attn(self.qkv, self.k_pool(l), self.v_pool(l), self.page_table, self.L, self.parent,
                         self.k_scale[l], self.v_scale[l], out=self.attn, ld_q=self.qkv.stride(0), T=T,
                         Hq=I.N_Q_HEADS)
            nv.quantize(self.attn, out=self.q_a.out, act=self.q_a.buf, canonical=False)
            self._note(s0 + 1, self.q_a)
            g_a = self.q_a.g
        self._linear(self.q_a.buf, g_a, lay["o"], self.h, residual=self.h)
        nv.rmsnorm_quantize(self.h, self.norm_w[2 * l + 1], self.eps, self.q_h.out, act=self.q_h.buf,
                            g_in=self._site(s0 + 2))
        self._note(s0 + 2, self.q_h)
        if self.static:
            # gate+up, SwiGLU and its NVFP4 with the site's static scale in one launch
            gu = lay["gate_up"]
            g_f = self._site(s0 + 3)
            nv.linear_swiglu(self.q_h.buf, self.q_h.g, T, gu.prep, gu.g, gu.N // 2, gu.K, g_f, self.q_f.buf)
        else:
            self._linear(self.q_h.buf, self.q_h.g, lay["gate_up"], self.gu)
            nv.swiglu_quantize(self.gu, self.q_f.out, act=self.q_f.buf)
            self._note(s0 + 3, self.q_f)
            g_f = self.q_f.g
        self._linear(self.q_f.buf, g_f, lay["down"], self.h, residual=self.h)

    def head(self):
        i = self.n_layers * self.SITES
        nv.rmsnorm_quantize(self.h, self.norm_w[-1], self.eps, self.q_h.out, act=self.q_h.buf, g_in=self._site(i))
        self._note(i, self.q_h)
        self._linear(self.q_h.buf, self.q_h.g, self.lm_head, self.logits)
        nv.argmax(self.logits, self.ids)

    def accept(self, draft_tokens):
        """Greedy acceptance after a step (self.ids = the target's token after each
        node) and compaction of the accepted tokens' K/V next to the context in
        every layer.  Returns device tensors (path, n_accepted, next_token)."""
        out = nv.tree_accept(draft_tokens, self.ids, self.parent)
        k0, v0 = self.kv[0, 0], self.kv[0, 1]
        nv.kv_compact(k0.data_ptr(), v0.data_ptr(), self.kv[0].nbytes, self.n_layers, I.N_KV_HEADS, I.HEAD_DIM,
                      self.n_pool, I.PAGE, self.page_table, self.L, out[0], out[1], self.T)
        return out

    def _linear(self, act, g, lin, y, residual=None, M=None):
        nv.linear(act, g, self.T if M is None else M, lin.prep, lin.g, lin.N, lin.K, y=y, residual=residual)

    # ------------------------------------------------------------------ prefill
    def _prefill_buffers(self, S):
        """Per-suffix buffers, kept for later calls of up to the same length:
        the bf16 activations of all S rows, one tile-image buffer for the
        widest K (reused by every quantisation site, whose quantiser writes it
        directly), and the head's one-row operands."""
        pf = getattr(self, "_pf", None)
        if pf is not None and pf["cap"] >= S:
            return pf
        H, F, Hq, Hkv, D = I.HIDDEN, I.FFN, I.N_Q_HEADS, I.N_KV_HEADS, I.HEAD_DIM
        cap = max(S, 1)
        kmax = max(H, F, Hq * D)
        dev = self.dev
        pf = {
            "cap": cap,
            "qkv": torch.empty(cap, (Hq + 2 * Hkv) * D, dtype=torch.bfloat16, device=dev),
            "attn": torch.empty(cap, Hq * D, dtype=torch.bfloat16, device=dev),
            "gu": torch.empty(cap, 2 * F, dtype=torch.bfloat16, device=dev),
            "g": torch.empty(1, dtype=torch.float32, device=dev),
            "wide": torch.empty(nv.prepared_weight_bytes(cap, kmax), dtype=torch.uint8, device=dev),
            "q_h": Act(H, dev),
            "streams": [torch.cuda.Stream(device=dev) for _ in range(PREFILL_STREAMS)]
            if dev.type == "cuda" else [],
            "logits": torch.empty(1, I.VOCAB, dtype=torch.bfloat16, device=dev),
            "ids": torch.empty(1, dtype=torch.int32, device=dev),
        }
        self._pf = pf
        return pf

    def prefill(self, h: torch.Tensor, start: int, layers=None):
        """Prefill the S = h.shape[0] suffix tokens at positions start .. start+S-1.

        h: bf16 [S, HIDDEN] (contiguous, on the model's device) holds the
        tokens' input hidden states and is overwritten with the last layer's
        output.  Every layer's K/V of the suffix lands in the paged FP8 cache
        (positions start .. in the page table), so that a verify step at
        ctx_len = start + S sees it.  Returns the device int32 [1] argmax of
        the last token's logits (the token that follows the suffix), or None
        without an LM head or for S == 0.

        layers: the layers to run, in order (default all); the head runs only
        when they end with the last layer.  Running range(0, k) and then
        range(k, n_layers) gives the same result as one call.

        Needs static activation scales (calibrate()): one calibrated tensor
        scale per quantisation site, as in the verify step.

        Per layer: RMSNorm + NVFP4 over all S rows, the QKV linear over all
        rows, the FP8 append of all S tokens' K/V, then causal attention in
        blocks of 128 queries (block b attends to the context, start + 128 b
        tokens, the earlier blocks included, plus its own causal chain), the
        attention output quantised with its site scale, the O linear (+h),
        RMSNorm + NVFP4, gate+up, SwiGLU + NVFP4, down (+h)."""
        if not self.static:
            raise RuntimeError("prefill needs static activation scales: call calibrate() first")
        S = h.shape[0]
        if h.dtype != torch.bfloat16 or h.dim() != 2 or h.shape[1] != I.HIDDEN or not h.is_contiguous():
            raise ValueError("h must be a contiguous bf16 [S, HIDDEN] tensor")
        if h.device.type != self.dev.type or (self.dev.index is not None and h.device.index != self.dev.index):
            raise ValueError(f"h is on {h.device}, the model on {self.dev}")
        if start < 0 or start + S > self.n_log * I.PAGE:
            raise ValueError(f"positions {start} .. {start + S - 1} exceed the page table "
                             f"({self.n_log} pages of {I.PAGE})")
        layers = range(self.n_layers) if layers is None else list(layers)
        if any(not 0 <= l < self.n_layers for l in layers):
            raise ValueError("layer index out of range")
        if S == 0:
            return None
        pf = self._prefill_buffers(S)
        qd = I.N_Q_HEADS * I.HEAD_DIM
        kd = I.N_KV_HEADS * I.HEAD_DIM
        qkv, attn, gu = pf["qkv"][:S], pf["attn"][:S], pf["gu"][:S]
        wide, g = pf["wide"], pf["g"]
        for l in layers:
            lay, s0 = self.layers[l], l * self.SITES
            kp, vp = self.k_pool(l), self.v_pool(l)
            # each quantiser writes the tile image the wide linear streams
            nv.rmsnorm_quantize_tiles(h, self.norm_w[2 * l], self.eps, self._site(s0), wide, g)
            self._wide(wide, g, lay["qkv"], qkv)
            nv.kv_append(qkv[:, qd:], qkv[:, qd + kd:], qkv.stride(0), S, kp, vp, self.page_table, start,
                         self.k_scale[l], self.v_scale[l])
            self._causal_blocks(pf, l, qkv, attn, start, S)
            nv.quantize_tiles(attn, self._site(s0 + 1), wide, g)
            self._wide(wide, g, lay["o"], h, residual=h)
            nv.rmsnorm_quantize_tiles(h, self.norm_w[2 * l + 1], self.eps, self._site(s0 + 2), wide, g)
            self._wide(wide, g, lay["gate_up"], gu)
            nv.swiglu_quantize_tiles(gu, self._site(s0 + 3), wide, g)
            self._wide(wide, g, lay["down"], h, residual=h)
        if self.lm_head is None or len(layers) == 0 or layers[-1] != self.n_layers - 1:
            return None
        i = self.n_layers * self.SITES
        a = pf["q_h"]
        nv.rmsnorm_quantize(h[S - 1:S], self.norm_w[-1], self.eps, a.out, act=a.buf, g_in=self._site(i))
        self._linear(a.buf, a.g, self.lm_head, pf["logits"], M=1)
        nv.argmax(pf["logits"], pf["ids"])
        return pf["ids"]

    def _causal_blocks(self, pf, l, qkv, attn, start, S):
        """The layer's causal attention, one call per block of 128 queries.  The
        blocks are independent once every suffix token's K/V is appended, so on
        the GPU they go round PREFILL_STREAMS streams (each with its own
        workspace), forked from and joined back into the current stream: one
        block's start overlaps another's tail."""
        kp, vp = self.k_pool(l), self.v_pool(l)
        chunks = prefill_chunks(start, S)
        k = min(len(pf["streams"]), len(chunks))
        if k < 2:
            for r, t, ctx in chunks:
                nv.causal_attn(qkv[r:r + t], kp, vp, self.page_table, ctx, self.k_scale[l], self.v_scale[l],
                               out=attn[r:r + t], ld_q=qkv.stride(0), T=t, Hq=I.N_Q_HEADS)
            return
        main = torch.cuda.current_stream(self.dev)
        fork = torch.cuda.Event()
        fork.record(main)
        splits = self._causal_splits(len(chunks))
        with nv.option(nv.OPT_ATTN_SPLITS, splits) if splits else contextlib.nullcontext():
            for i, (r, t, ctx) in enumerate(chunks):
                s = pf["streams"][i % k]
                if i < k:
                    s.wait_event(fork)
                with torch.cuda.stream(s):
                    nv.causal_attn(qkv[r:r + t], kp, vp, self.page_table, ctx, self.k_scale[l], self.v_scale[l],
                                   out=attn[r:r + t], ld_q=qkv.stride(0), T=t, Hq=I.N_Q_HEADS,
                                   ws=nv.default_workspace("attn", i % k))
        for s in pf["streams"][:k]:
            join = torch.cuda.Event()
            join.record(s)
            main.wait_event(join)

    def _causal_splits(self, n_blocks):
        """Context splits per query head that the prefill gives each causal
        call: PREFILL_ATTN_SPLITS while at least 4 blocks run at once on the
        streams, else 0 (the library's own count, which fills the GPU with one
        call).  With several calls in flight, fewer and longer CTAs pay the
        per-CTA query setup, split write-out and combine fewer times (on B200,
        8 blocks of a 942-token suffix: 471 us per layer at 3 splits on 8
        streams against 517 us at the library's 6).  A split count the caller
        set through OPT_ATTN_SPLITS stands."""
        k = min(PREFILL_STREAMS, n_blocks) if self.dev.type == "cuda" else 1
        if k < 4 or nv.get_option(nv.OPT_ATTN_SPLITS) > 0:
            return 0
        return PREFILL_ATTN_SPLITS

    def _wide(self, act, g, lin, y, residual=None):
        nv.linear_wide(act, g, y.shape[0], lin.prep, lin.g, lin.N, lin.K, y=y, residual=residual)

    def turn(self, h_suffix: torch.Tensor, draft_tokens: torch.Tensor | None = None):
        """One agent turn's forward work: restore the reused prefix pages,
        prefill the suffix (the S = ctx_len - prefix_tokens positions the
        restore does not hold; h_suffix is overwritten), then verify the tree
        in self.h / self.parent at ctx_len, and with draft tokens accept the
        longest matching path.  Needs static activation scales (calibrate()),
        as prefill() does.  Returns (token after the suffix, ids of the verify
        step, and the acceptance tuple of accept() or None)."""
        S = h_suffix.shape[0]
        if S != self.L - self.prefix_tokens:
            raise ValueError(f"the suffix has {self.L - self.prefix_tokens} tokens after the "
                             f"{self.prefix_tokens}-token prefix, got {S}")
        self.restore()
        nxt = self.prefill(h_suffix, self.prefix_tokens)
        self.step(restore=False)
        acc = self.accept(draft_tokens) if draft_tokens is not None else None
        return nxt, self.ids, acc

    def prefill_launches(self, S):
        """Kernel launches of prefill(S rows): per layer norm-q, qkv, K/V
        append, one causal attention call per block of 128 queries
        (nv.attn_launches() launches each, at the split count the blocks
        run at), quantise, o, norm-q, gate_up,
        swiglu-q, down (each quantiser writes the wide linear's tile image);
        then the head on the last row."""
        n = len(prefill_chunks(0, S))
        splits = self._causal_splits(n)
        if splits:
            sms = torch.cuda.get_device_properties(self.dev).multi_processor_count
            per_call = nv.attn_launches(splits * I.N_Q_HEADS, sms)
        else:
            per_call = nv.attn_launches()
        return 0 if S == 0 else self.n_layers * (9 + n * per_call) + \
            (self.LAUNCHES_HEAD if self.lm_head is not None else 0)

    def step(self, restore=True):
        """One verify step on the current self.h / self.parent; result in self.ids."""
        if restore:
            self.restore()
        for l in range(self.n_layers):
            self.layer(l)
        if self.lm_head is not None:
            self.head()

    LAUNCHES_HEAD = 3                # norm-q, lm head, argmax

    @property
    def launches_per_layer(self):
        """norm-q, qkv, kv-append, attention (nv.attn_launches(): split and
        combine, or one with the fused combine), [quantise], o, norm-q,
        gate_up, [swiglu-q], down (with static scales the attention output is
        quantised in the combine and the SwiGLU in the gate+up launch)."""
        return (7 if self.static else 9) + nv.attn_launches()

    def launches_per_step(self, restore=True):
        return (1 if restore else 0) + self.n_layers * self.launches_per_layer + \
            (self.LAUNCHES_HEAD if self.lm_head is not None else 0)

    # ------------------------------------------------------------------ bytes
    def linear_bytes(self):
        """Algorithmic HBM bytes of all linear launches in one step: weight codes
        + scales, activation codes + scales, bf16 outputs (+ residual reads);
        with static scales the gate+up launch writes the NVFP4 SwiGLU output
        (N/2 features) instead of the bf16 gate and up."""
        T, tot = self.T, 0
        for lay in self.layers:
            for name, lin in lay.items():
                out = T * (lin.N // 2) * 9 // 16 if (name == "gate_up" and self.static) else T * lin.N * 2
                tot += lin.nbytes + T * lin.K * 9 // 16 + out * (2 if name in ("o", "down") else 1)
        if self.lm_head is not None:
            lin = self.lm_head
            tot += lin.nbytes + T * lin.K * 9 // 16 + T * lin.N * 2
        return tot

    def attn_bytes(self):
        """K + V bytes read per step (context + tree slots, all layers)."""
        return self.n_layers * 2 * (self.L + self.T) * I.N_KV_HEADS * I.HEAD_DIM

    def restore_bytes(self):
        return 2 * self.src_ids.numel() * PAGE_BYTES          # read + write

    def step_bytes(self, restore=True):
        return self.linear_bytes() + self.attn_bytes() + (self.restore_bytes() if restore else 0)
