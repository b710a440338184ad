"""fp64 oracle of a packed batch whose sequences interleave video and text segments.

TEST INFRASTRUCTURE ONLY (imported by tests/ and nothing else). It never imports the CUDA
package and the CUDA package never imports it.

The hybrid scheme gives video tokens Native Sparse Attention and text tokens dense
attention (shd-paper.top page "VideoNSA: Native Sparse Attention Scales Video
Understanding", abstract); clip lengths vary from request to request (CSDN blog on
VideoNSA, vcloud.csdn.net, section 5.2, item 3). The pages never place text between video
segments; the plainest reading that keeps both rules, and reduces to the trailing-text
layout, is the one computed here, sequence by sequence:

  * video rows: NSA over the sequence's video tokens only, taken in order as one stream
    (text tokens are skipped): compression blocks, selection blocks, the window and the
    causal masks all count positions in that stream, exactly as a sequence made of those
    video tokens alone;
  * text rows: dense causal softmax attention over every earlier token of the sequence,
    video and text, and the row itself; gates are not used.

Both halves are evaluated by the single-sequence oracle (oracle.prefill_rows): the video
stream as an all-video sequence, and the text rows as the dense rows of the whole sequence
(n_video = 0, where every row is dense causal).
"""
from __future__ import annotations

from dataclasses import replace

import numpy as np

from oracle import oracle as orc


def segments_of(cu_seqlens, seg_lens, seg_video):
    """Per sequence, the list of (start, length, is_video) segments, positions absolute in
    the packed batch. seg_lens / seg_video list the segments in packed order; they must tile
    every sequence exactly."""
    cu = [int(x) for x in cu_seqlens]
    out, pos, si = [], 0, 0
    for b in range(len(cu) - 1):
        segs = []
        while pos < cu[b + 1]:
            ln = int(seg_lens[si])
            if ln <= 0 or pos + ln > cu[b + 1]:
                raise ValueError("segments must have positive lengths and stay inside their sequence")
            segs.append((pos, ln, bool(seg_video[si])))
            pos += ln
            si += 1
        out.append(segs)
    if si != len(seg_lens):
        raise ValueError("more segments than tokens")
    return out


def video_positions(segs):
    """Absolute positions of a sequence's video tokens, in stream order."""
    return np.array([p for (s, ln, vid) in segs if vid for p in range(s, s + ln)], dtype=np.int64)


def text_positions(segs):
    return np.array([p for (s, ln, vid) in segs if not vid for p in range(s, s + ln)], dtype=np.int64)


def packed_prefill(cfg: orc.OracleConfig, q, k, v, gates, cu_seqlens, seg_lens, seg_video, nthreads: int = 0,
                   sel_override=None):
    """Every row of a packed batch. q [N, hq, d], k/v [N, hkv, d] (bf16 bit patterns), gates
    [N, hq, 3] float32; cfg carries the heads and NSA constants (its n_tokens / n_video are
    ignored). sel_override, if given, is the selection of every video row in stream order
    (sequence after sequence), as the GPU reports it; the selected branch then uses it.

    Returns {"out": [N, hq, d] fp64, "sel": [Nv, hkv, n] int32, "scores": list per sequence
    of [nv_b, hkv, Nsel_b], "video_rows": positions of the video rows in stream order}."""
    per_seq = segments_of(cu_seqlens, seg_lens, seg_video)
    N = int(cu_seqlens[-1])
    out = np.zeros((N, cfg.hq, cfg.d))
    sels, scores, vrows = [], [], []
    done = 0
    for b, segs in enumerate(per_seq):
        s0, s1 = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        if s1 == s0:
            continue
        vp = video_positions(segs)
        tp = text_positions(segs)
        if len(vp):
            cv = replace(cfg, n_tokens=len(vp), n_video=len(vp))
            so = None
            if sel_override is not None:
                so = sel_override[done: done + len(vp)]
            o = orc.prefill_rows(cv, q[vp], k[vp], v[vp], gates[vp], np.arange(len(vp), dtype=np.int32),
                                 sel_override=so, nthreads=nthreads)
            out[vp] = o["out"]
            sels.append(o["sel"])
            scores.append(o["scores"])
            vrows.append(vp)
            done += len(vp)
        if len(tp):
            ct = replace(cfg, n_tokens=s1 - s0, n_video=0)
            o = orc.prefill_rows(ct, q[s0:s1], k[s0:s1], v[s0:s1], gates[s0:s1], (tp - s0).astype(np.int32),
                                 want=(), nthreads=nthreads)
            out[tp] = o["out"]
    empty_sel = np.zeros((0, cfg.hkv, cfg.top_n), dtype=np.int32)
    return {"out": out, "sel": np.concatenate(sels) if sels else empty_sel, "scores": scores,
            "video_rows": np.concatenate(vrows) if vrows else np.zeros(0, dtype=np.int64)}
