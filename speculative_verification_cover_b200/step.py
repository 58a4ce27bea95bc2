"""One verification step over device-resident buffers, built on the C ABI.

A step is the four library calls in order, on one stream:
  1. dd_dualview_attention  -- dual-view attention (one layer, or each layer of a
                               stack, optionally after a cached prefix) with d_in, d_out
  2. dd_verify_logits       -- per-row statistics and coupled samples
  3. dd_select_seeds        -- the next step's seed set from u, d_in, d_out
  4. dd_decide              -- KEEP / REPLACE / REMASK
Buffers are allocated once (torch, caller side); the library itself never
allocates. The step (and each of its three phases) can be captured into CUDA graphs and replayed.
"""
from __future__ import annotations

import torch

from . import dd
from .workloads import WorkloadSpec

INPUT_KEYS = ("q", "k_cur", "v_cur", "k_prev", "v_prev", "is_seed", "is_masked", "is_new",
              "eligible", "tokens", "logits_t", "logits_d")
# Our kernels per step: per attention layer mask preparation, pass 1, pass 2 and
# the head reduction; vocabulary stream + merge; seed selection; decisions.
KERNELS_PER_LAYER = 4
KERNELS_PER_STEP = KERNELS_PER_LAYER + 4  # one attention layer


class VerifyStep:
    def __init__(self, spec: WorkloadSpec, inputs: dict, seed: int = 2024, step_index: int = 1,
                 use_seeds: bool = True, extra_layers=(), prefix_cache: bool = False):
        """extra_layers: attention operands (q, k_cur, v_cur, k_prev, v_prev) of further
        layers after the one in `inputs`; the step then runs every layer, averaging d_in
        and d_out over them. prefix_cache: the prompt's K/V rows are a cache filled
        once, so every layer computes the query rows after the prompt only."""
        self.spec = spec
        self.x = {k: inputs[k] for k in INPUT_KEYS}
        self.extra_layers = list(extra_layers)
        self.q_begin = spec.prompt if prefix_cache else 0
        dev = self.x["q"].device
        B, L, Hq, Hkv, d, R = spec.B, spec.L, spec.Hq, spec.Hkv, spec.d, spec.R
        self.seed, self.step_index = seed, step_index
        self.use_seeds = use_seeds and spec.k > 0
        self.out = torch.empty_like(self.x["q"])
        self.lse = torch.empty(B, Hq, L, device=dev)
        self.d_in = torch.empty(B, L, device=dev)
        self.d_out = torch.empty(B, L, device=dev)
        self.ws = torch.empty(dd.dd_dualview_attention_workspace_size(B, L, Hq, Hkv, d),
                              dtype=torch.uint8, device=dev)
        self.stats = dd.RowStats.empty(B, R, dev)
        self.vws = torch.empty(dd.dd_verify_logits_workspace_size(B, R, spec.V,
                                                                  self.x["logits_t"].dtype),
                               dtype=torch.uint8, device=dev)
        self.k = max(spec.k, 1)
        self.next_seeds = torch.empty(B, self.k, dtype=torch.int32, device=dev)
        self.next_is_seed = torch.empty(B, L, dtype=torch.uint8, device=dev)
        self.score = torch.empty(B, L, device=dev)
        self.decision = torch.empty(B, L, dtype=torch.uint8, device=dev)
        self.new_tokens = torch.empty(B, L, dtype=torch.int32, device=dev)
        self.accepted = torch.empty(B, dtype=torch.uint8, device=dev)
        self.graphs = None
        self.side = None
        # recorded by the attention call right after its mask preparation (forked())
        self.prep_done = torch.cuda.Event()
        with torch.cuda.device(dev):
            self.prep_done.record()  # creates the event on the inputs' device

    @property
    def n_layers(self):
        return 1 + len(self.extra_layers)

    @property
    def kernels_per_step(self):
        return KERNELS_PER_LAYER * self.n_layers + 4

    # --- the four calls
    def attention(self, prep_done=None):
        x, n = self.x, self.n_layers
        for li, y in enumerate([x] + self.extra_layers):
            dd.dd_dualview_attention_ex(
                y["q"], y["k_cur"], y["v_cur"], y["k_prev"] if self.use_seeds else None,
                y["v_prev"] if self.use_seeds else None, x["is_seed"] if self.use_seeds else None,
                x["is_masked"], x["is_new"], self.out, self.lse, self.d_in, self.d_out, self.ws,
                q_begin=self.q_begin, accumulate_stats=li > 0, stats_weight=1.0 / n,
                prep_done=prep_done if li == 0 else None)

    def verify(self):
        s = self.spec
        dd.dd_verify_logits(self.x["logits_t"], self.x["logits_d"], self.stats,
                            pos_offset=s.pos_offset, temperature=s.temperature, seed=self.seed,
                            step=self.step_index, workspace=self.vws)

    def select(self):
        s, x = self.spec, self.x
        dd.dd_select_seeds(self.stats.entropy_t, s.pos_offset, self.d_in, self.d_out,
                           x["eligible"], self.next_seeds, self.next_is_seed, self.score)

    def decide(self):
        s, x = self.spec, self.x
        dd.dd_decide(s.policy, x["tokens"], x["is_seed"], x["eligible"], self.stats,
                     s.pos_offset, self.decision, self.new_tokens, self.accepted,
                     tau_kl=s.tau_kl, tau_conf=s.tau_conf, temperature=s.temperature)

    def select_and_decide(self):
        self.select()
        self.decide()

    def __call__(self):
        self.attention()
        self.verify()
        self.select_and_decide()

    def forked(self):
        """The same step on two streams. The attention call runs on the main stream; the
        vocabulary pass and then the decisions (they read only its statistics) run on a
        side stream that starts once the attention's mask preparation is done: by then
        the first attention pass holds its SMs (the preparation releases it early), and
        the vocabulary pass, whose CTAs take chunks of work as they become free, fills
        every other SM and then the pass's SMs as they empty. Started together instead,
        the vocabulary pass would take every SM and the attention would wait for it.
        Seed selection needs both, so it waits for the vocabulary pass's event and runs
        beside the decisions."""
        main = torch.cuda.current_stream()
        if self.side is None:
            self.side = torch.cuda.Stream(device=main.device)
            self.verified = torch.cuda.Event()
        self.attention(prep_done=self.prep_done)
        with torch.cuda.stream(self.side):
            self.side.wait_event(self.prep_done)
            self.verify()
            self.verified.record(self.side)
            self.decide()
        main.wait_event(self.verified)
        self.select()
        main.wait_stream(self.side)

    def choose_initial_seeds(self):
        """Pass 0 with an empty seed set, then the stability score picks the seeds the
        step will verify (the seeds of step t come from the scores of step t-1)."""
        if self.spec.k == 0:
            return
        keep = self.use_seeds
        self.use_seeds = False
        self.attention()
        self.verify()
        s = self.spec
        dd.dd_select_seeds(self.stats.entropy_t, s.pos_offset, self.d_in, self.d_out,
                           self.x["eligible"], self.next_seeds, self.next_is_seed, self.score)
        self.x["is_seed"].copy_(self.next_is_seed)
        self.use_seeds = keep

    # --- CUDA graphs
    def capture(self):
        """Capture the step as one CUDA graph (what a serving loop replays; the
        vocabulary pass runs beside the attention call) and, for the per-phase
        breakdown, each of the three phases as a graph of its own."""
        self()  # warm every kernel (lazy attribute set-up happens outside capture)
        torch.cuda.synchronize()
        graphs = []
        for fn in (self.attention, self.verify, self.select_and_decide):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            graphs.append(g)
        whole = torch.cuda.CUDAGraph()
        with torch.cuda.graph(whole):
            self.forked()
        graphs.append(whole)
        torch.cuda.synchronize()
        self.graphs = graphs
        return graphs

    def replay(self, events=None):
        """Replay the step. Without events: the one-graph step. With 4 timing events:
        the three phase graphs, with the events recorded before attention, before
        verify, after verify and at the end (the events between phases cost a few
        microseconds of their own)."""
        ga, gv, gs, whole = self.graphs
        if not events:
            whole.replay()
            return
        events[0].record()
        ga.replay()
        events[1].record()
        gv.replay()
        events[2].record()
        gs.replay()
        events[3].record()

    def result_tensors(self):
        """What a caller reads back after a step."""
        return (self.decision, self.new_tokens, self.accepted, self.next_seeds)
