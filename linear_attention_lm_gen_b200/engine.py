"""A chunked-prefill serving loop over the JetBlock mixer with a state and
history cache.

The recurrent state of a JetBlock layer has a fixed size per sequence (its
H x dv x dk float32 state and the last three raw values of V for the conv),
which is what makes the mixer cheap to serve: the Jet-Nemotron paper (section
2.5, finding 4; the efficiency FAQ of the explainer) puts decode speed down to
cache size. This module keeps those per-sequence states in two pools and runs
the library's calls on them:

  admit(seq)   take a free pool entry (zero state and history)
  prefill(seq, ...)  the sequence's next prompt tokens, in pieces of at most
               `chunk_tokens` (chunked prefill), each piece continuing from
               the entry's state and history (jet_jetblock_prefill)
  prefill_many({seq: ...})  the same for several sequences of different
               lengths: in every round, the pieces of all of them run as one
               variable-length call (jet_jetblock_prefill_varlen; shapes off
               the tensor-core path batch pieces of equal length instead)
  decode(seqs, ...)  one new token for each of a batch of sequences, in place
               on their entries (jet_jetblock_decode_slots)
  release(seq) return the entry
  submit(seq, prompt) / step(tokens)  a serving iteration: up to
               `chunk_tokens` queued prompt tokens (oldest prompt first; a
               long prompt continues in later steps), then one decode token
               for each running sequence the caller supplies a token for

All arithmetic runs in the library's kernels. This module only keeps the
pool bookkeeping and orders the calls. torch provides device memory and
moves data: it stacks the pieces of a batched call and gathers and scatters
their pool entries (the prefill takes its states as one [B,...] tensor).
Everything is issued on torch's current stream, so the library calls and
the data movement stay in order.
"""
from __future__ import annotations

import torch

from . import (jet_jetblock_decode_slots, jet_jetblock_prefill, jet_jetblock_prefill_varlen,
               jet_jetblock_prefill_workspace_size)

MAX_VARLEN_SEQS = 256    # sequences per variable-length call


class JetEngine:
    def __init__(self, W1: torch.Tensor, W2: torch.Tensor, H: int, dk: int, dv: int, max_seqs: int,
                 chunk_tokens: int = 4096):
        if chunk_tokens <= 0 or max_seqs <= 0:
            raise ValueError("chunk_tokens and max_seqs must be positive")
        self.W1, self.W2 = W1, W2
        self.H, self.dk, self.dv = H, dk, dv
        self.chunk_tokens = chunk_tokens
        dev, dt = W1.device, W1.dtype
        self.S = torch.zeros((max_seqs, H, dv, dk), device=dev, dtype=torch.float32)
        self.hist = torch.zeros((max_seqs, 3, H, dv), device=dev, dtype=dt)
        self._hist_out = torch.empty((1, 3, H, dv), device=dev, dtype=dt)
        self._free = list(range(max_seqs - 1, -1, -1))    # pop() hands out the lowest entry first
        self.slot: dict = {}                               # sequence id -> pool entry
        self.pos: dict = {}                                # sequence id -> tokens consumed
        self._ws = None
        self._queue: list = []                             # [seq, prompt tuple, tokens done]

    # ---------------------------------------------------------------- pool entries
    @property
    def free_slots(self) -> int:
        return len(self._free)

    def admit(self, seq) -> int:
        """Give `seq` a pool entry with a zero state and a zero history."""
        if seq in self.slot:
            raise KeyError(f"sequence {seq!r} is already admitted")
        if not self._free:
            raise RuntimeError("state cache is full")
        s = self._free.pop()
        self.S[s].zero_()
        self.hist[s].zero_()
        self.slot[seq] = s
        self.pos[seq] = 0
        return s

    def release(self, seq) -> None:
        self._free.append(self.slot.pop(seq))
        del self.pos[seq]

    # ---------------------------------------------------------------- the mixer
    def pieces(self, T: int):
        """Token ranges of a prompt of T tokens, at most chunk_tokens each."""
        return [(t0, min(T, t0 + self.chunk_tokens)) for t0 in range(0, T, self.chunk_tokens)]

    def _workspace(self, T: int, B: int = 1):
        n = jet_jetblock_prefill_workspace_size(B, T, self.H, self.dk, self.dv, 64, self.W1.dtype)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(max(n, 16), device=self.W1.device, dtype=torch.uint8)
        return self._ws

    def prefill(self, seq, x, q, k, v, g, beta) -> torch.Tensor:
        """The next T prompt tokens of `seq`: x [T,D], q, k [T,H,dk], v [T,H,dv]
        (raw), g, beta [T,H]. Returns o [T,H,dv]; the entry's state and history
        advance past the tokens."""
        s = self.slot[seq]
        S = self.S[s:s + 1]
        outs = []
        for t0, t1 in self.pieces(x.shape[0]):
            piece = lambda a: a[t0:t1].unsqueeze(0)
            o, _ = jet_jetblock_prefill(piece(x), self.W1, self.W2, piece(q), piece(k), piece(v), piece(g),
                                        piece(beta), self.hist[s:s + 1], self._hist_out, S, None, S,
                                        self._workspace(t1 - t0))
            self.hist[s].copy_(self._hist_out[0])
            outs.append(o[0])
            self.pos[seq] += t1 - t0
        return torch.cat(outs) if len(outs) > 1 else outs[0]

    @property
    def varlen(self) -> bool:
        """Whether prefill_many can pack pieces of different lengths into one
        call (the variable-length prefill takes the tensor-core shapes)."""
        return self.W1.dtype == torch.bfloat16 and self.dk in (64, 96, 128) and self.dv % 128 == 0

    def prefill_many(self, prompts: dict) -> dict:
        """Chunked prefill of several sequences at once. prompts: seq ->
        (x, q, k, v, g, beta) as for prefill (lengths may differ). Round r
        takes the r-th piece of every sequence that has one; all of them run
        as one variable-length call (packed along the token axis), or, off the
        tensor-core shapes, pieces of equal length share one batched call.
        Returns seq -> o [T,H,dv]."""
        outs = {seq: [] for seq in prompts}
        plan = {seq: self.pieces(inp[0].shape[0]) for seq, inp in prompts.items()}
        for r in range(max((len(p) for p in plan.values()), default=0)):
            groups: dict = {}
            if self.varlen:
                live = [seq for seq, p in plan.items() if r < len(p)]
                for i in range(0, len(live), MAX_VARLEN_SEQS):
                    self._prefill_packed(prompts, plan, r, live[i:i + MAX_VARLEN_SEQS], outs)
                continue
            for seq, p in plan.items():
                if r < len(p):
                    groups.setdefault(p[r][1] - p[r][0], []).append(seq)
            for L, seqs in groups.items():
                idx = torch.tensor([self.slot[sq] for sq in seqs], device=self.S.device)
                S = self.S.index_select(0, idx)
                hin = self.hist.index_select(0, idx)
                hout = torch.empty_like(hin)
                stack = [torch.stack([prompts[sq][j][plan[sq][r][0]:plan[sq][r][1]] for sq in seqs])
                         for j in range(6)]
                o, _ = jet_jetblock_prefill(stack[0], self.W1, self.W2, *stack[1:], hin, hout, S, None, S,
                                            self._workspace(L, len(seqs)))
                self.S.index_copy_(0, idx, S)
                self.hist.index_copy_(0, idx, hout)
                for b, sq in enumerate(seqs):
                    outs[sq].append(o[b])
                    self.pos[sq] += L
        return {sq: torch.cat(v) if len(v) > 1 else v[0] for sq, v in outs.items()}

    def _prefill_packed(self, prompts, plan, r, seqs, outs):
        """Round r's pieces of `seqs` as one variable-length call."""
        lens = [plan[sq][r][1] - plan[sq][r][0] for sq in seqs]
        cu = [0]
        for n in lens:
            cu.append(cu[-1] + n)
        idx = torch.tensor([self.slot[sq] for sq in seqs], device=self.S.device)
        S = self.S.index_select(0, idx)
        hin = self.hist.index_select(0, idx)
        hout = torch.empty_like(hin)
        packed = [torch.cat([prompts[sq][j][plan[sq][r][0]:plan[sq][r][1]] for sq in seqs]) for j in range(6)]
        o, _ = jet_jetblock_prefill_varlen(packed[0], self.W1, self.W2, *packed[1:], cu, hin, hout, S, None, S)
        self.S.index_copy_(0, idx, S)
        self.hist.index_copy_(0, idx, hout)
        for i, sq in enumerate(seqs):
            outs[sq].append(o[cu[i]:cu[i + 1]])
            self.pos[sq] += lens[i]

    # ---------------------------------------------------------------- serving iterations
    def submit(self, seq, prompt) -> None:
        """Queue a prompt (x, q, k, v, g, beta as for prefill); the sequence is
        admitted now, so the cache must have a free entry."""
        if len(prompt) != 6 or prompt[0].shape[0] == 0:
            raise ValueError("a prompt is (x, q, k, v, g, beta) of at least one token")
        if any(a.shape[0] != prompt[0].shape[0] for a in prompt):
            raise ValueError("the arrays of a prompt must have the same number of tokens")
        self.admit(seq)
        self._queue.append([seq, prompt, 0])

    @property
    def prefilling(self) -> list:
        return [q[0] for q in self._queue]

    def step(self, tokens: dict | None = None) -> dict:
        """One serving iteration. Prefill: up to chunk_tokens tokens of the
        queued prompts, oldest first (prefill_many batches pieces of equal
        length). Decode: one token for every sequence in `tokens` (seq ->
        (x, q, k, v, g, beta) of one token), which must have finished its
        prompt. Returns seq -> outputs of this step ([n,H,dv] prompt outputs
        for prefill, [H,dv] for a decoded token)."""
        budget, work, took = self.chunk_tokens, {}, {}
        for seq, prompt, done in self._queue:
            if budget == 0:
                break
            n = min(budget, prompt[0].shape[0] - done)
            work[seq] = tuple(a[done:done + n] for a in prompt)
            took[seq] = n
            budget -= n
        still = {seq for seq, prompt, done in self._queue if done + took.get(seq, 0) < prompt[0].shape[0]}
        # every check comes before any work is issued
        unknown = [sq for sq in (tokens or ()) if sq not in self.slot]
        if unknown:
            raise KeyError(f"decode tokens for sequences that are not admitted: {sorted(map(str, unknown))}")
        busy = still & set(tokens or ())
        if busy:
            raise ValueError(f"sequences still in prefill: {sorted(map(str, busy))}")
        out = self.prefill_many(work) if work else {}
        for item in self._queue:
            item[2] += took.get(item[0], 0)
        self._queue = [q for q in self._queue if q[0] in still]
        if tokens:
            seqs = list(tokens)
            stack = [torch.stack([tokens[sq][j] for sq in seqs]) for j in range(6)]
            o = self.decode(seqs, *stack)
            for b, sq in enumerate(seqs):
                out[sq] = o[b]
        return out

    def decode(self, seqs, x, q, k, v, g, beta) -> torch.Tensor:
        """One new token for each sequence of `seqs` (batch order): x [B,D],
        q, k [B,H,dk], v [B,H,dv] (raw), g, beta [B,H]. Returns o [B,H,dv]."""
        if len(set(seqs)) != len(seqs):
            raise ValueError("a sequence appears twice in one decode batch")
        unknown = [sq for sq in seqs if sq not in self.slot]
        if unknown:
            raise KeyError(f"sequences that are not admitted: {sorted(map(str, unknown))}")
        slots = torch.tensor([self.slot[s] for s in seqs], dtype=torch.int32).to(self.S.device, non_blocking=True)
        o = jet_jetblock_decode_slots(x, self.W1, self.W2, q, k, v, g, beta, self.hist, self.S, slots)
        for s in seqs:
            self.pos[s] += 1
        return o
