"""Pipeline trace of the tensor-core attention kernel.

    python -m ulysses_sequence_attention_sp_b200.trace --workload vit

Builds the library with -DUSP_TRACE (into libusp_trace.so beside libusp.so),
runs the named workload's Ulysses block a few times on random inputs, and
prints the clock64() stamps that CTA 7 recorded at each pipeline event, per
key tile, relative to its first "S ready". The kernel counts key tiles over
all the items a persistent CTA walks, so consecutive rows may belong to
different items; the per-item table shows the hand-off between items.

Events (one stamp per key tile unless marked per item):
  Kload    producer: K of the next tile issued
  Vload    producer: V of this tile issued
  QKiss    MMA: Q K^T of this tile issued
  PVstart  MMA: P of this tile seen (p_full)
  PViss    MMA: P V of this tile issued
  Sready   softmax: S of this tile ready (warp 0)
  Sld      softmax: S loaded from TMEM
  maxx     softmax: row maxima exchanged
  exps     softmax: exponentials, sums and packing done
  Parr     softmax: P stored and p_full arrived
  combine  per item: denominators combined
  o_full   per item: the last P V has completed
  epi_done per item: the epilogue's stores issued
"""

from __future__ import annotations

import argparse
import ctypes
import os
import sys

import numpy as np

EVENTS, TILES = 14, 256
TILE_EVENTS = ["Kload", "Vload", "QKiss", "PVstart", "PViss", "Sready", "Sld", "maxx", "exps", "Parr"]
ITEM_EVENTS = {10: "combine", 11: "o_full", 12: "epi_done"}


def main(argv=None) -> int:
    from . import build, workloads

    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="vit", choices=[w.name.split("-")[0] for w in workloads.ALL])
    ap.add_argument("--num-chunks", type=int, default=1)
    ap.add_argument("--tiles", type=int, default=30, help="key tiles to print")
    args = ap.parse_args(argv)
    lib_path = os.path.join(os.path.dirname(build.LIB_PATH), "libusp_trace.so")
    build.build(extra=["-DUSP_TRACE"], out=lib_path)
    os.environ["USP_LIBRARY"] = lib_path  # read when usp loads the library

    import torch
    from . import usp

    w = next(x for x in workloads.ALL if x.name.split("-")[0] == args.workload)
    if w.dtype not in ("bf16", "fp16"):
        print(f"{w.name}: the tensor-core kernel runs 16-bit inputs only", file=sys.stderr)
        return 2
    plan = usp.Plan(w.batch, w.seq_len, w.heads, w.head_dim, w.world, w.dtype, w.prefix, kv_heads=w.heads_kv,
                    ring_size=w.ring)
    q = [t.normal_() for t in plan.empty_seq_shards()]
    k, v = ([t.normal_() for t in plan.empty_kv_seq_shards()] for _ in range(2))
    out = plan.empty_seq_shards()
    ws = torch.empty(plan.workspace_bytes(args.num_chunks), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        usp.ulysses_attention(plan, q, k, v, out=out, num_chunks=args.num_chunks, workspace=ws)
    torch.cuda.synchronize()
    if usp.device_status() != 0:
        print("a device-side wait ran out", file=sys.stderr)
        return 1
    lib = ctypes.CDLL(lib_path)
    buf = (ctypes.c_ulonglong * (EVENTS * TILES))()
    if lib.usp_debug_read_trace(buf, EVENTS * TILES) != 0:
        print("could not read the trace", file=sys.stderr)
        return 1
    tr = np.array(buf, dtype=np.int64).reshape(EVENTS, TILES)
    base = tr[5, 0]
    ntiles = int(np.sum(tr[5] > 0))
    print(f"{w.name}, num_chunks={args.num_chunks}: clk relative to the first S ready of CTA 7")
    print("tile " + " ".join(f"{n:>8s}" for n in TILE_EVENTS))
    for j in range(min(args.tiles, ntiles)):
        print(f"{j:4d} " + " ".join(f"{tr[e, j] - base:8d}" for e in range(len(TILE_EVENTS))))
    items = int(np.sum(tr[10] > 0))
    if items:
        print("item " + " ".join(f"{n:>8s}" for n in ITEM_EVENTS.values()))
        for it in range(min(items, 16)):
            print(f"{it:4d} " + " ".join(f"{tr[e, it] - base:8d}" for e in ITEM_EVENTS))
    sl = slice(min(2, ntiles - 1), max(min(ntiles, 120), 3))
    if ntiles > 4:
        print("median period per tile (S ready to S ready):", float(np.median(np.diff(tr[5, sl]))))
    plan.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
