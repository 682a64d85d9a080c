"""A whole decode step as one CUDA graph.

One step of serving is: upload the step's new K/V tokens and queries from
pinned host buffers, quantize-append the tokens, run decode attention, and
download the output. Issued call by call that is a dozen host calls
(copies, the append and its length advance, the split-K pass and its merge),
each with its launch latency; captured once into a CUDA graph it is one
launch. Every kernel in it is the library's; the graph only replays them.
"""
from __future__ import annotations

from . import _binding as B


class DecodeStep:
    """Capture the decode step over fixed buffers; `run()` replays it.

    k_host, v_host: pinned host [n_new][H][128] (bf16, fp16 or fp32), the
    step's new tokens in cu_new order; q_host: pinned host [S][Hq][128];
    the caller refills them before every run. When k_host, v_host and q_host
    lie back to back in one pinned buffer (k, then v, then q, each a multiple
    of 16 bytes), the step uploads them with one copy instead of three.
    seq_lens, cu_new: device int32
    (seq_lens advances by the appended tokens on every run). The output lands
    in `out_host` (pinned fp32 [S][Hq][128]) once the stream is synchronized.

    max_seq_len is fixed at capture: a replay that took a sequence past it
    would make attention leave out its newest tokens (the kernels clamp and
    flag KVQ_DEV_SEQLEN in the status word). So the step counts its replays
    against the lengths it last read and `run()` raises before one would
    overflow; after changing seq_lens by other means, call `sync_lengths()`.
    """

    def __init__(self, desc, seq_lens, cu_new, max_seq_len: int, softmax_scale: float, k_host, v_host,
                 q_host, out_host=None, workspace=None):
        import torch
        dev = seq_lens.device
        for t, name in ((k_host, "k_host"), (v_host, "v_host"), (q_host, "q_host")):
            if t.is_cuda or not t.is_pinned():
                raise ValueError("%s must be pinned host memory" % name)
        self.desc, self.seq_lens, self.cu_new = desc, seq_lens, cu_new
        self.max_seq_len, self.scale = max_seq_len, float(softmax_scale)
        self.k_host, self.v_host, self.q_host = k_host, v_host, q_host
        parts = (k_host, v_host, q_host)
        self.h_all = None
        if (all(t.is_contiguous() for t in parts) and k_host.nbytes % 16 == 0 and v_host.nbytes % 16 == 0
                and all(a.untyped_storage().data_ptr() == b.untyped_storage().data_ptr()
                        and a.data_ptr() + a.nbytes == b.data_ptr() for a, b in zip(parts, parts[1:]))):
            # one upload: the three as byte ranges of one host and one device buffer
            total = sum(t.nbytes for t in parts)
            base = k_host.storage_offset() * k_host.element_size()
            self.h_all = torch.empty(0, dtype=torch.uint8).set_(k_host.untyped_storage(), base, (total,))
            self.d_all = torch.empty(total, dtype=torch.uint8, device=dev)
            views, off = [], 0
            for t in parts:
                views.append(self.d_all[off:off + t.nbytes].view(t.dtype).view(t.shape))
                off += t.nbytes
            self.dk, self.dv, self.dq = views
        else:
            self.dk = torch.empty(k_host.shape, dtype=k_host.dtype, device=dev)
            self.dv = torch.empty(v_host.shape, dtype=v_host.dtype, device=dev)
            self.dq = torch.empty(q_host.shape, dtype=q_host.dtype, device=dev)
        S, Hq = q_host.shape[0], q_host.shape[1]
        self.out = torch.empty((S, Hq, 128), dtype=torch.float32, device=dev)
        self.out_host = out_host if out_host is not None else torch.empty(
            (S, Hq, 128), dtype=torch.float32).pin_memory()
        need = B.decode_workspace_size(desc, S, Hq, max_seq_len)
        self.ws = workspace if workspace is not None else torch.empty(max(need, 16), dtype=torch.uint8,
                                                                      device=dev)
        # One eager decode (no state change) does the library's per-variant
        # set-up outside the capture.
        B.decode_attention(desc, self.dq, seq_lens, max_seq_len, self.scale, out=self.out, workspace=self.ws)
        torch.cuda.synchronize(dev)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        self.graph = torch.cuda.CUDAGraph()
        # thread-local capture: other threads of the process (a process group's
        # watchdog, for one) may keep making CUDA calls meanwhile
        with torch.cuda.graph(self.graph, stream=side, capture_error_mode="thread_local"):
            self._body()
        torch.cuda.current_stream(dev).wait_stream(side)
        self.sync_lengths()

    def sync_lengths(self) -> None:
        """Read seq_lens and cu_new (one device synchronization) and recount
        the replays left before a sequence would pass max_seq_len."""
        lens = self.seq_lens.cpu().tolist()
        cu = self.cu_new.cpu().tolist()
        left = None
        for s, t in enumerate(lens):
            inc = cu[s + 1] - cu[s]
            if inc > 0:
                n = max(0, (self.max_seq_len - t) // inc)
                left = n if left is None else min(left, n)
        self.replays_left = left  # None: no sequence grows

    def _body(self):
        if self.h_all is not None:
            self.d_all.copy_(self.h_all, non_blocking=True)
        else:
            self.dk.copy_(self.k_host, non_blocking=True)
            self.dv.copy_(self.v_host, non_blocking=True)
            self.dq.copy_(self.q_host, non_blocking=True)
        B.quantize_append(self.desc, self.dk, self.dv, self.cu_new, self.seq_lens)
        B.decode_attention(self.desc, self.dq, self.seq_lens, self.max_seq_len, self.scale, out=self.out,
                           workspace=self.ws)
        self.out_host.copy_(self.out, non_blocking=True)

    def run(self) -> None:
        """Replay the step on the current stream (asynchronous). Raises
        before a replay would take a sequence past max_seq_len."""
        if self.replays_left is not None:
            if self.replays_left <= 0:
                raise RuntimeError("DecodeStep: the next replay would take a sequence past max_seq_len=%d "
                                   "(call sync_lengths() after changing seq_lens)" % self.max_seq_len)
            self.replays_left -= 1
        self.graph.replay()
