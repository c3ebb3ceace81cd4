"""Decode-step driver: runs ODA steps of a synthetic workload through the C ABI.

One step, in the order of the method notes ("On-Demand Attention：让语言模型按需读取完整历史")
§2.3, issued on one stream with no host synchronisation:

  local pass : per layer oda_attend_local (S^L) or the recurrent stand-in; oda_glue_hidden -> h^L
               [hybrid: the recurrent layers read state buffer i and write buffer 1 - i]
  oda_recall_score(h_{t-1}, E(x_t), h^L) -> score, flag, any_flag
  oda_cond_begin(any_flag)          # a CUDA-graph IF node when captured
     full pass: per layer oda_attend_full_if (S^F, flagged sequences only); glue -> h^F
               [hybrid: the recurrent layers read the untouched pre-step buffer i again]
  oda_cond_end
  oda_commit(flag): chosen branch's staged K,V -> cache slot of position t, h_{t-1} <- h^b, t += 1

All compute is in liboda.so; this module only allocates buffers (torch), fills the seeded
inputs (workload/) and issues the calls.  Per-step inputs live in one flat byte buffer
(``StepLayout``) so that staging a step is a single copy (device-to-device for the kernel
benchmark, pinned host-to-device for the end-to-end one).
"""
from __future__ import annotations

import numpy as np
import torch

from workload import configs, device as wdev, inputs
from workload.configs import Workload

from . import oda

LOCAL, FULL = 0, 1


class StepLayout:
    """Offsets of one step's inputs inside a flat, 256-byte aligned byte buffer."""

    def __init__(self, wl: Workload):
        B, L, Hq, Hkv, D = wl.B, wl.L, wl.Hq, wl.Hkv, wl.D
        G = len(wl.gdn_layers)
        if wl.backbone:
            # q/k/v come from the backbone's projections and E(x_t) from the previous step's LM
            # head: a step's only host input is the schedule
            ent = [("sched", (B,), torch.int32)]
        else:
            ent = [("q", (2, L, B, Hq, 128), torch.bfloat16), ("k", (2, L, B, Hkv, 128), torch.bfloat16),
                   ("v", (2, L, B, Hkv, 128), torch.bfloat16), ("emb", (B, D), torch.float32),
                   ("sched", (B,), torch.int32)]
        if G:
            ent += [("gc", (2, G, B, configs.CONV_WIDTH), torch.float32),
                    ("gv", (2, G, B, configs.GDN_HEADS, configs.GDN_DIM), torch.float32),
                    ("ga", (2, G, B, configs.GDN_HEADS), torch.float32),
                    ("gb", (2, G, B, configs.GDN_HEADS), torch.float32)]
        self.entries = []
        off = 0
        for name, shape, dt in ent:
            nbytes = int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
            self.entries.append((name, shape, dt, off, nbytes))
            off += (nbytes + 255) // 256 * 256
        self.nbytes = off

    def views(self, buf: torch.Tensor) -> dict:
        out = {}
        for name, shape, dt, off, nbytes in self.entries:
            out[name] = buf[off:off + nbytes].view(dt).view(shape)
        return out


def fill_step_inputs(wl: Workload, step: int, views: dict) -> None:
    """Writes step ``step``'s seeded inputs into device views (bit-identical to the host
    generator: q/k/v by the device generator, fp32 inputs generated on the host)."""
    sched = inputs.schedule(wl, step)
    views["sched"].copy_(torch.from_numpy(sched if sched is not None else np.zeros(wl.B, np.int32)))
    if wl.backbone:
        return
    for br in (LOCAL, FULL):
        for a, layer in enumerate(wl.attn_layers):
            kq, kk, kv = inputs.qkv_keys(wl, step, layer, br)
            wdev.fill_normal_bf16(views["q"][br, a], kq)
            wdev.fill_normal_bf16(views["k"][br, a], kk)
            wdev.fill_normal_bf16(views["v"][br, a], kv)
    views["emb"].copy_(torch.from_numpy(inputs.emb(wl, step)))
    for br in (LOCAL, FULL):
        for j, layer in enumerate(wl.gdn_layers):
            c, v, a, b = inputs.gdn_step_inputs(wl, step, layer, br)
            views["gc"][br, j].copy_(torch.from_numpy(c))
            views["gv"][br, j].copy_(torch.from_numpy(v))
            views["ga"][br, j].copy_(torch.from_numpy(a))
            views["gb"][br, j].copy_(torch.from_numpy(b))


class OdaDecoder:
    """Device state of one workload (paged caches, positions, h_{t-1}, head weights, hybrid
    state) plus the call sequence of one decode step."""

    def __init__(self, wl: Workload, device="cuda", capacity_steps: int = 0,
                 perturb_head: bool = False, head_params: dict = None, fill_cache: bool = True,
                 overlap_layers: bool = True, deterministic: bool = False, kv_format: str = "bf16",
                 bb_fused: bool = True):
        if not torch.cuda.is_available():
            raise RuntimeError("OdaDecoder needs a CUDA device (the CUDA path has no fallback)")
        self.wl = wl
        self.bb_fused = bb_fused
        dev = torch.device(device)
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        torch.cuda.set_device(self.device)
        B, L, Hkv, D = wl.B, wl.L, wl.Hkv, wl.D
        self.capacity_steps = max(wl.steps, capacity_steps)
        self.max_pages = (max(wl.ctx) + self.capacity_steps + 1 + configs.PAGE - 1) // configs.PAGE
        self.n_pool = B * self.max_pages
        cfg = oda.make_config(B, wl.Hq, Hkv, self.max_pages, D, wl.sinks, wl.window, wl.theta,
                              overlap_layers=overlap_layers, deterministic=deterministic)
        self.ctx = oda.oda_create(cfg)
        dev = self.device
        self.stream = torch.cuda.Stream(dev)
        self.page_table = torch.from_numpy(inputs.page_table(wl, self.max_pages)).to(dev)
        if kv_format not in ("bf16", "fp8"):
            raise ValueError("kv_format must be 'bf16' or 'fp8'")
        self.kv_format = kv_format
        self.k_pool, self.v_pool, self.kv8_pool = [], [], []
        for a in range(L):
            k = torch.empty((self.n_pool, Hkv, configs.PAGE, 128), dtype=torch.bfloat16, device=dev)
            v = torch.empty_like(k)
            if fill_cache:
                wdev.fill_kv(k, self.page_table, wl.ctx,
                             [inputs.cache_key(wl, "k", a, b) for b in range(B)], Hkv)
                wdev.fill_kv(v, self.page_table, wl.ctx,
                             [inputs.cache_key(wl, "v", a, b) for b in range(B)], Hkv)
            if kv_format == "bf16":
                self.k_pool.append(k)
                self.v_pool.append(v)
            else:
                # the seeded bf16 cache of this layer, packed into fp8 page blocks by the library
                kv8 = torch.empty((self.n_pool, Hkv, oda.KV8_BLOCK_BYTES), dtype=torch.uint8, device=dev)
                oda.oda_kv8_pack(oda.kv_layer(k, v), oda.kv8_layer(kv8), Hkv)
                torch.cuda.synchronize(dev)
                self.kv8_pool.append(kv8)
                del k, v
        if kv_format == "bf16":
            self.layers = [oda.kv_layer(self.k_pool[a], self.v_pool[a]) for a in range(L)]
        else:
            self.layers = [oda.kv8_layer(self.kv8_pool[a]) for a in range(L)]
        fp8 = kv_format == "fp8"
        self._attend_local = oda.oda_attend_local_fp8 if fp8 else oda.oda_attend_local
        self._attend_full = oda.oda_attend_full_if_fp8 if fp8 else oda.oda_attend_full_if
        self._commit = oda.oda_commit_fp8 if fp8 else oda.oda_commit
        self.pos = torch.tensor([c + 1 for c in wl.ctx], dtype=torch.int32, device=dev)
        # the step's results (h_{t-1} after the commit, q_t, the routing flags) share one
        # device block, so they come back to the host in a single copy (read_results)
        self.results = torch.zeros(B * D + 2 * B, dtype=torch.float32, device=dev)
        self.h_prev = self.results[:B * D].view(B, D)
        self.h_prev.copy_(torch.from_numpy(inputs.h_prev0(wl)))
        hp = head_params if head_params is not None else inputs.head_weights(wl, perturb_head)
        self.head_params = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for k, v in hp.items()}
        self.head_w = oda.head_weights(self.head_params)
        n_layers = wl.n_layers
        self.o = torch.zeros((2, n_layers, B, D), dtype=torch.float32, device=dev)
        self.h = torch.zeros((2, B, D), dtype=torch.float32, device=dev)
        self.score = self.results[B * D:B * D + B]
        self.flag = self.results[B * D + B:].view(torch.int32)
        self.any_flag = torch.zeros(1, dtype=torch.int32, device=dev)
        self.layout = StepLayout(wl)
        # Two staging buffers, used by alternate steps (and one captured graph each): host inputs
        # of step i + 1 are uploaded on a copy stream into the buffer step i does not read, so
        # the upload overlaps step i's kernels.
        self.staging = [torch.zeros(self.layout.nbytes, dtype=torch.uint8, device=dev)
                        for _ in range(2)]
        self.svs = [self.layout.views(b) for b in self.staging]
        self.slot = 0
        self._n_staged = 0
        self.copy_stream = torch.cuda.Stream(dev)
        self.staged = [torch.cuda.Event() for _ in range(2)]
        self.released = [torch.cuda.Event() for _ in range(2)]
        self.routing_scheduled = wl.routing == "bernoulli"
        self._n_launched = 0
        if wl.hybrid:
            # two state buffers used alternately (ping-pong): a step reads the pre-step recurrent
            # and conv state from one and writes the advanced state to the other, so the full
            # retry reads the untouched pre-step state directly - no snapshot or restore copies
            S0, C0 = inputs.gdn_state0(wl)
            self.rec_buf = [torch.from_numpy(S0).to(dev), torch.empty(S0.shape, dtype=torch.float32, device=dev)]
            self.conv_buf = [torch.from_numpy(C0).to(dev), torch.empty(C0.shape, dtype=torch.float32, device=dev)]
            self.states = [oda.state(self.rec_buf[i], self.conv_buf[i]) for i in range(2)]
            self.taps = torch.from_numpy(
                np.stack([inputs.gdn_taps(wl, layer) for layer in wl.gdn_layers])).to(dev)
        if wl.backbone:
            self._init_backbone()
        self.graph = None
        torch.cuda.synchronize(dev)

    def _init_backbone(self) -> None:
        """Seeded random weights of the synthetic backbone (bf16 projections filled on the device,
        bit-identical to workload.inputs), its buffers, and E(x_1) of the first tokens."""
        wl, dev = self.wl, self.device
        B, D, F, V, L = wl.B, wl.D, wl.ffn, wl.vocab, wl.L
        shapes = inputs.bb_shapes(wl)
        fill_stream = torch.cuda.current_stream(dev)   # the device fills run on torch's stream

        def packed(R, C, key, log2_scale):
            """A seeded N(0,1) * 2^log2_scale matrix, generated row-major, stored packed."""
            tmp = torch.empty((R, C), dtype=torch.bfloat16, device=dev)
            wdev.fill_normal_bf16(tmp, key, 0, log2_scale)
            out = torch.empty_like(tmp)
            oda.oda_bb_pack_weight(self.ctx, tmp, out, fill_stream)
            return out

        self.bb_w, self.bb_layers = [], []
        for a, layer in enumerate(wl.attn_layers):
            ws = {}
            for name in inputs.BB_TENSORS:
                R, C = shapes[name]
                ws[name] = packed(R, C, inputs.bb_weight_key(wl, layer, name), inputs.bb_log2_scale(C))
            ga, gm = inputs.bb_norms(wl, layer)
            ws["attn_norm"] = torch.from_numpy(ga).to(dev)
            ws["mlp_norm"] = torch.from_numpy(gm).to(dev)
            self.bb_w.append(ws)
            self.bb_layers.append(oda.bb_layer(ws["attn_norm"], ws["w_qkv"], ws["w_o"], ws["mlp_norm"],
                                               ws["w_gate"], ws["w_up"], ws["w_down"]))
        self.bb_final_norm = torch.from_numpy(inputs.bb_norms(wl, -1)[0]).to(dev)
        self.bb_embed = packed(V, D, inputs.bb_embed_key(wl), inputs.BB_EMBED_LOG2_SCALE)
        fill_stream.synchronize()
        self.bb_x = torch.zeros((2, B, D), dtype=torch.float32, device=dev)
        self.bb_act = torch.zeros((B, F), dtype=torch.bfloat16, device=dev)
        self.bb_logits = torch.zeros((B, V), dtype=torch.float32, device=dev)
        self.bb_q = torch.zeros((2, L, B, wl.Hq, 128), dtype=torch.bfloat16, device=dev)
        self.bb_k = torch.zeros((2, L, B, wl.Hkv, 128), dtype=torch.bfloat16, device=dev)
        self.bb_v = torch.zeros_like(self.bb_k)
        self.token = torch.from_numpy(inputs.bb_token0(wl)).to(dev)
        self.emb = torch.zeros((B, D), dtype=torch.float32, device=dev)
        oda.oda_bb_embed(self.ctx, self.bb_embed, V, self.token, self.emb, self.stream)
        self.stream.synchronize()

    def backbone_bytes(self) -> int:
        """Weight bytes one backbone pass streams (projections of every layer)."""
        return sum(t.numel() * t.element_size() for ws in self.bb_w
                   for n, t in ws.items() if n.startswith("w_"))

    # ---------------------------------------------------------------- inputs
    def make_step_buffer(self, step: int) -> torch.Tensor:
        buf = torch.zeros(self.layout.nbytes, dtype=torch.uint8, device=self.device)
        fill_step_inputs(self.wl, step, self.layout.views(buf))
        return buf

    @property
    def sv(self) -> dict:
        """Views of the staging buffer of the most recently staged step."""
        return self.svs[self.slot]

    def stage(self, src: torch.Tensor) -> None:
        """Copies one step's input buffer into the next staging buffer.  A device buffer is
        copied in the step stream's order; a (pinned) host buffer is uploaded on the copy stream
        once the step that last read that staging buffer has run, so the upload overlaps the
        previous step.  The caller keeps a host buffer unchanged until its step has run."""
        self.slot = self._n_staged % 2
        self._n_staged += 1
        i, dst = self.slot, self.staging[self.slot]
        self.stream.wait_stream(torch.cuda.current_stream(self.device))
        if src.is_cuda:
            # an elementwise copy on the SMs (a device-to-device memcpy runs on a copy engine at a
            # fraction of the bandwidth); int32 lanes keep every bit
            with torch.cuda.stream(self.stream):
                torch.bitwise_or(src.view(torch.int32), 0, out=dst.view(torch.int32))
            return
        self.copy_stream.wait_event(self.released[i])
        with torch.cuda.stream(self.copy_stream):
            dst.copy_(src, non_blocking=True)
            self.staged[i].record(self.copy_stream)
        self.stream.wait_event(self.staged[i])

    # ------------------------------------------------------------------ step
    def _bb_pass(self, br: int, stream, flag=None) -> None:
        """One backbone pass of branch br: the residual starts from E(x_t); every layer projects
        q/k/v from it, attends (S^L or, for flagged sequences, S^F), adds o_proj and the MLP;
        then the final norm gives h^br."""
        wl, ctx = self.wl, self.ctx
        x = self.bb_x[br]
        n_attn = len(wl.attn_layers)
        oda.oda_bb_begin(ctx, self.emb, x, stream)
        oda.oda_bb_qkv(ctx, self.bb_layers[0], x, self.bb_q[br, 0], self.bb_k[br, 0], self.bb_v[br, 0],
                       stream)
        for a, layer in enumerate(wl.attn_layers):
            q, k, v = self.bb_q[br, a], self.bb_k[br, a], self.bb_v[br, a]
            if br == LOCAL:
                self._attend_local(ctx, self.layers[a], self.page_table, self.pos, q, k, v,
                                   self.o[br, layer], stream)
            else:
                self._attend_full(ctx, self.layers[a], self.page_table, self.pos, flag, q, k, v,
                                  self.o[br, layer], stream)
            last = a + 1 == n_attn
            if self.bb_fused:   # o_proj, the MLP and the next layer's QKV in one launch
                nq = (None, None, None) if last else (self.bb_q[br, a + 1], self.bb_k[br, a + 1],
                                                      self.bb_v[br, a + 1])
                oda.oda_bb_post_attention(ctx, self.bb_layers[a], None if last else self.bb_layers[a + 1],
                                          self.o[br, layer], x, self.bb_act, *nq, stream=stream)
            else:
                oda.oda_bb_attn_out(ctx, self.bb_layers[a], self.o[br, layer], x, stream)
                oda.oda_bb_mlp(ctx, self.bb_layers[a], x, self.bb_act, stream)
                if not last:
                    oda.oda_bb_qkv(ctx, self.bb_layers[a + 1], x, self.bb_q[br, a + 1],
                                   self.bb_k[br, a + 1], self.bb_v[br, a + 1], stream)
        oda.oda_bb_final_norm(ctx, self.bb_final_norm, x, self.h[br], stream)

    def _issue_backbone(self) -> None:
        """One decode step of the whole synthetic model: local pass, recall head, conditional full
        pass, commit, then the LM head on the committed hidden state (its greedy token's embedding
        is E(x_{t+1}) of the next step)."""
        wl, s, sv, ctx = self.wl, self.stream, self.sv, self.ctx
        self._bb_pass(LOCAL, s)
        oda.oda_recall_score(ctx, self.head_w, self.h_prev, self.emb, self.h[LOCAL],
                             sv["sched"] if self.routing_scheduled else None, self.score,
                             self.flag, self.any_flag, s)
        body = oda.oda_cond_begin(ctx, s, self.any_flag)
        self._bb_pass(FULL, body, self.flag)
        oda.oda_cond_end(ctx, s)
        self._commit(ctx, self.layers, self.page_table, self.pos, self.flag, self.bb_k[LOCAL],
                     self.bb_v[LOCAL], self.bb_k[FULL], self.bb_v[FULL], self.h[LOCAL], self.h[FULL],
                     self.h_prev, s)
        oda.oda_bb_lm_head(ctx, self.bb_embed, wl.vocab, self.h_prev, self.bb_logits, self.token,
                           self.emb, s)

    def issue_always_full(self) -> None:
        """The reference decoder the method is measured against: every step one backbone pass with
        full attention in every layer for every sequence, no local pass and no recall head, then
        the commit of that pass and the LM head (synthetic-backbone workloads only)."""
        wl, s, ctx = self.wl, self.stream, self.ctx
        if not hasattr(self, "ones"):
            self.ones = torch.ones(wl.B, dtype=torch.int32, device=self.device)
        self._bb_pass(FULL, s, self.ones)
        self._commit(ctx, self.layers, self.page_table, self.pos, self.ones, self.bb_k[FULL],
                     self.bb_v[FULL], self.bb_k[FULL], self.bb_v[FULL], self.h[FULL], self.h[FULL],
                     self.h_prev, s)
        oda.oda_bb_lm_head(ctx, self.bb_embed, wl.vocab, self.h_prev, self.bb_logits, self.token,
                           self.emb, s)

    def issue(self) -> None:
        """Enqueues one decode step on self.stream (eagerly or into a capture)."""
        if self.wl.backbone:
            self._issue_backbone()
            return
        wl, s, sv = self.wl, self.stream, self.sv
        ctx = self.ctx
        n_layers = wl.n_layers
        if wl.hybrid:   # the step with staging slot i reads state i and writes state 1 - i
            cur, nxt = self.states[self.slot], self.states[1 - self.slot]
        a = j = 0
        for layer in range(n_layers):
            if layer in wl.attn_layers:
                self._attend_local(ctx, self.layers[a], self.page_table, self.pos, sv["q"][LOCAL, a],
                                   sv["k"][LOCAL, a], sv["v"][LOCAL, a], self.o[LOCAL, layer], s)
                a += 1
            else:
                oda.oda_glue_gdn_step(ctx, cur, nxt, j, sv["gc"][LOCAL, j], sv["gv"][LOCAL, j],
                                      sv["ga"][LOCAL, j], sv["gb"][LOCAL, j], self.taps[j], None,
                                      self.o[LOCAL, layer], s)
                j += 1
        oda.oda_glue_hidden(ctx, sv["emb"], self.o[LOCAL], n_layers, None, self.h[LOCAL], s)
        oda.oda_recall_score(ctx, self.head_w, self.h_prev, sv["emb"], self.h[LOCAL],
                             sv["sched"] if self.routing_scheduled else None, self.score,
                             self.flag, self.any_flag, s)
        body = oda.oda_cond_begin(ctx, s, self.any_flag)
        a = j = 0
        for layer in range(n_layers):
            if layer in wl.attn_layers:
                self._attend_full(ctx, self.layers[a], self.page_table, self.pos, self.flag,
                                  sv["q"][FULL, a], sv["k"][FULL, a], sv["v"][FULL, a],
                                  self.o[FULL, layer], body)
                a += 1
            else:
                # flagged sequences: from the pre-step state, over the local pass's result
                oda.oda_glue_gdn_step(ctx, cur, nxt, j, sv["gc"][FULL, j], sv["gv"][FULL, j],
                                      sv["ga"][FULL, j], sv["gb"][FULL, j], self.taps[j], self.flag,
                                      self.o[FULL, layer], body)
                j += 1
        oda.oda_glue_hidden(ctx, sv["emb"], self.o[FULL], n_layers, self.flag, self.h[FULL], body)
        oda.oda_cond_end(ctx, s)
        self._commit(ctx, self.layers, self.page_table, self.pos, self.flag, sv["k"][LOCAL],
                     sv["v"][LOCAL], sv["k"][FULL], sv["v"][FULL], self.h[LOCAL], self.h[FULL],
                     self.h_prev, s)

    def capture(self) -> None:
        """Records one step (with the retry under a conditional node) as a CUDA graph, once per
        staging buffer."""
        torch.cuda.synchronize(self.device)
        graphs, slot = [], self.slot
        for i in range(2):
            self.slot = i
            oda.oda_graph_begin(self.stream)
            try:
                self.issue()
            except Exception:
                try:
                    oda.oda_graph_end(self.stream).close()
                except Exception:
                    pass
                for g in graphs:
                    g.close()
                self.slot = slot
                raise
            graphs.append(oda.oda_graph_end(self.stream))
        self.slot = slot
        self.graph = graphs

    def live_state(self):
        """(recurrent, conv) buffers holding the state after the last launched step (hybrid)."""
        i = self._n_launched % 2
        return self.rec_buf[i], self.conv_buf[i]

    def launch(self) -> None:
        """Runs one step on the most recently staged inputs."""
        if self.wl.hybrid and self.slot != self._n_launched % 2:
            raise RuntimeError("hybrid steps alternate their state buffers with the staging "
                               "buffers: stage new inputs before every step")
        self._n_launched += 1
        if self.graph is not None:
            self.graph[self.slot].launch(self.stream)
        else:
            self.issue()
        self.released[self.slot].record(self.stream)

    def step(self, src: torch.Tensor = None) -> None:
        if src is not None:
            self.stage(src)
        self.launch()

    def read_results(self, out: torch.Tensor) -> None:
        """Copies the last step's results (h_prev [B][D], then score [B], then flag [B] as
        int32 bits) into `out`, a pinned float32 host tensor of B*D + 2B elements, in the step
        stream's order (asynchronous: synchronize before reading it)."""
        with torch.cuda.stream(self.stream):
            out.copy_(self.results, non_blocking=True)

    def synchronize(self):
        self.stream.synchronize()

    def device_error(self) -> int:
        self.synchronize()
        return oda.oda_get_error(self.ctx)

    def attention_layers_bytes(self) -> int:
        if self.kv_format == "fp8":
            return sum(p.numel() for p in self.kv8_pool)
        return sum(k.numel() * 2 * 2 for k in self.k_pool)

    def close(self):
        if self.graph is not None:
            for g in self.graph:
                g.close()
            self.graph = None
        self.ctx.close()
