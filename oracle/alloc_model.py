"""Reference model of the paged KV block manager -- TEST INFRASTRUCTURE.

A plain dictionary model of the lifecycle on "vLLM 與 PagedAttention：高吞吐推理
的關鍵", section 三 (運作流程): a new request gets an empty block table and no
blocks up front (step 一); prefill writes its tokens block by block and takes
a new block each time one fills (step 二); each decoded token goes into the
current block, or into a new block when the current one is full (step 三);
when the request ends all of its blocks go back to the pool for any other
request (step 四).  Section 二 fixes the block size (16 tokens) and the table
(logical block i -> physical block); sharing (section 二, "無法共享"): several
tables may point at the same physical blocks.  Reference counts are how
"shared" and "freed on completion" fit together: a block returns to the pool
when the last table that holds it lets go.

Readings where the pages are silent:
  * the initial free list is a caller-given permutation of [0, NB); blocks are
    taken from its front and freed blocks are appended to its back;
  * ``fork(parent, child, n)`` gives the child the parent's first n tokens by
    sharing the blocks that hold them (refcount + 1 each); n defaults to the
    parent's length;
  * appending into a partly filled last block that other tables also hold is a
    copy-on-write: the sequence takes a fresh block in its place and the pair
    (shared block, fresh block) is queued for the caller to copy on the device
    (beam candidates share prefix blocks -- "vllm", PagedAttention 的核心原理);
  * swap space (P3 section 二 2.2, --swap-space): a sequence whose blocks are
    all unshared can be moved to host slots (its GPU blocks return to the
    pool) and later back into fresh GPU blocks; the moves are queued as
    (GPU block, host slot) pairs; while out it can only come back or be freed;
  * every failing call leaves the state exactly as it was.
"""
from __future__ import annotations

from collections import deque

BLOCK_TOKENS = 16


class AllocError(Exception):
    def __init__(self, kind: str, msg: str = ""):
        super().__init__(f"{kind}: {msg}")
        self.kind = kind  # "invalid" | "oom" | "unsupported"


def blocks_for(n_tokens: int) -> int:
    return -(-n_tokens // BLOCK_TOKENS)


class BlockManager:
    def __init__(self, num_blocks: int, free_order=None):
        self.num_blocks = int(num_blocks)
        order = list(range(self.num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(self.num_blocks)):
            raise AllocError("invalid", "free order must be a permutation of the pool")
        self.free = deque(order)
        self.ref = [0] * self.num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.copies: list[tuple[int, int]] = []
        self.host_free: deque = deque()
        self.swapped: set = set()
        self.moves = {0: [], 1: []}  # 0: out (gpu -> host), 1: in (host -> gpu)

    # -- lifecycle ---------------------------------------------------------
    def add_seq(self, seq_id: int, num_tokens: int) -> None:
        if seq_id in self.tables or num_tokens < 0:
            raise AllocError("invalid", "sequence exists or negative length")
        need = blocks_for(num_tokens)
        if need > len(self.free):
            raise AllocError("oom")
        blocks = [self.free.popleft() for _ in range(need)]
        for b in blocks:
            self.ref[b] = 1
        self.tables[seq_id] = blocks
        self.lens[seq_id] = num_tokens

    def append_token(self, seq_id: int) -> int:
        if seq_id not in self.tables or seq_id in self.swapped:
            raise AllocError("invalid", "unknown or swapped-out sequence")
        blocks, pos = self.tables[seq_id], self.lens[seq_id]
        if pos % BLOCK_TOKENS == 0:
            if not self.free:
                raise AllocError("oom")
            b = self.free.popleft()
            self.ref[b] = 1
            blocks.append(b)
        elif self.ref[blocks[-1]] > 1:  # copy-on-write of the shared last block
            if not self.free:
                raise AllocError("oom")
            b = self.free.popleft()
            self.ref[b] = 1
            self.ref[blocks[-1]] -= 1
            self.copies.append((blocks[-1], b))
            blocks[-1] = b
        self.lens[seq_id] = pos + 1
        return blocks[pos // BLOCK_TOKENS] * BLOCK_TOKENS + pos % BLOCK_TOKENS

    def append_tokens(self, seq_ids) -> list[int]:
        """One token for each listed sequence (one decode step), all or none:
        an unknown or repeated id, then a shortage of free blocks (fresh and
        copy-on-write blocks together) is reported before anything changes."""
        ids = list(seq_ids)
        if len(set(ids)) != len(ids) or any(s not in self.tables or s in self.swapped for s in ids):
            raise AllocError("invalid", "unknown or repeated sequence")
        need, released = 0, {}
        for s in ids:
            if self.lens[s] % BLOCK_TOKENS == 0:
                need += 1
            else:
                last = self.tables[s][-1]
                if self.ref[last] - released.get(last, 0) > 1:
                    released[last] = released.get(last, 0) + 1
                    need += 1
        if need > len(self.free):
            raise AllocError("oom")
        return [self.append_token(s) for s in ids]

    def take_copies(self):
        import numpy as np

        src = np.array([c[0] for c in self.copies], np.int64)
        dst = np.array([c[1] for c in self.copies], np.int64)
        self.copies = []
        return src, dst

    def extend(self, seq_id: int, n: int):
        """n more tokens (a prompt or a prefill chunk), all or none: step 二
        of the lifecycle -- a new block each time one fills."""
        import numpy as np

        if seq_id not in self.tables or seq_id in self.swapped or n < 0:
            raise AllocError("invalid", "unknown or swapped-out sequence")
        blocks, ln = self.tables[seq_id], self.lens[seq_id]
        cow = ln % BLOCK_TOKENS != 0 and self.ref[blocks[-1]] > 1 and n > 0
        need = int(cow) + blocks_for(ln + n) - len(blocks)
        if need > len(self.free):
            raise AllocError("oom")
        return np.array([self.append_token(seq_id) for _ in range(n)], np.int64)

    def fork(self, parent: int, child: int, num_tokens: int | None = None) -> None:
        if parent not in self.tables or parent in self.swapped or child in self.tables:
            raise AllocError("invalid", "unknown parent or existing child")
        n = self.lens[parent] if num_tokens is None or num_tokens < 0 else num_tokens
        if n > self.lens[parent]:
            raise AllocError("invalid", "fork longer than the parent")
        self.tables[child] = list(self.tables[parent][: blocks_for(n)])
        self.lens[child] = n
        for b in self.tables[child]:
            self.ref[b] += 1

    def free_seq(self, seq_id: int) -> None:
        if seq_id not in self.tables:
            raise AllocError("invalid", "unknown sequence")
        if seq_id in self.swapped:
            self.host_free.extend(self.tables.pop(seq_id))
            self.swapped.discard(seq_id)
        else:
            for b in self.tables.pop(seq_id):
                self.ref[b] -= 1
                if self.ref[b] == 0:
                    self.free.append(b)
        del self.lens[seq_id]

    def set_host_pool(self, n: int) -> None:
        if n < 0 or self.swapped:
            raise AllocError("invalid", "bad size or host slots in use")
        self.host_free = deque(range(n))

    def swap_out(self, seq_id: int) -> None:
        if seq_id not in self.tables or seq_id in self.swapped:
            raise AllocError("invalid", "unknown or swapped sequence")
        blocks = self.tables[seq_id]
        if any(self.ref[b] != 1 for b in blocks):
            raise AllocError("unsupported", "shared blocks stay on the GPU")
        if len(blocks) > len(self.host_free):
            raise AllocError("oom")
        slots = []
        for b in blocks:
            h = self.host_free.popleft()
            self.moves[0].append((b, h))
            self.ref[b] = 0
            self.free.append(b)
            slots.append(h)
        self.tables[seq_id] = slots
        self.swapped.add(seq_id)

    def swap_in(self, seq_id: int) -> None:
        if seq_id not in self.swapped:
            raise AllocError("invalid", "not swapped out")
        slots = self.tables[seq_id]
        if len(slots) > len(self.free):
            raise AllocError("oom")
        blocks = []
        for h in slots:
            b = self.free.popleft()
            self.ref[b] = 1
            self.moves[1].append((b, h))
            self.host_free.append(h)
            blocks.append(b)
        self.tables[seq_id] = blocks
        self.swapped.discard(seq_id)

    def take_swaps(self, direction: int):
        import numpy as np

        pairs, self.moves[direction] = self.moves[direction], []
        return (np.array([p[0] for p in pairs], np.int64), np.array([p[1] for p in pairs], np.int64))

    # -- views -------------------------------------------------------------
    def export(self, seq_ids, width: int):
        import numpy as np

        tables = np.full((len(seq_ids), width), -1, dtype=np.int32)
        lens = np.zeros(len(seq_ids), dtype=np.int32)
        for i, s in enumerate(seq_ids):
            if s not in self.tables or s in self.swapped:
                raise AllocError("invalid", "unknown or swapped-out sequence")
            blocks = self.tables[s]
            if len(blocks) > width:
                raise AllocError("invalid", "table wider than the export width")
            tables[i, : len(blocks)] = blocks
            lens[i] = self.lens[s]
        return tables, lens

    def free_blocks(self) -> list[int]:
        return list(self.free)

    def slot_of(self, seq_id: int, pos: int) -> int:
        if seq_id in self.swapped or not 0 <= pos < self.lens[seq_id]:
            raise AllocError("invalid", "position outside the sequence")
        return self.tables[seq_id][pos // BLOCK_TOKENS] * BLOCK_TOKENS + pos % BLOCK_TOKENS

    def prefix_groups(self, seq_ids):
        """Sequences sharing leading blocks: those whose first block is full and
        held by several tables, grouped by it (first-appearance order); the
        group's prefix is the longest run of leading blocks identical in, and
        full for, every member.  Returns (prefix_blocks, offsets, members) with
        members given as indices into seq_ids."""
        import numpy as np

        ids = list(seq_ids)
        if any(s not in self.tables or s in self.swapped for s in ids):
            raise AllocError("invalid", "unknown or swapped-out sequence")
        by_first: dict[int, list[int]] = {}
        for i, s in enumerate(ids):
            if self.lens[s] >= BLOCK_TOKENS and self.ref[self.tables[s][0]] >= 2:
                by_first.setdefault(self.tables[s][0], []).append(i)
        pb = np.zeros(len(ids), np.int32)
        offs, members = [0], []
        for grp in by_first.values():
            if len(grp) < 2:
                continue
            common = min(self.lens[ids[i]] // BLOCK_TOKENS for i in grp)
            t0 = self.tables[ids[grp[0]]]
            k = 0
            while k < common and all(self.tables[ids[i]][k] == t0[k] for i in grp):
                k += 1
            if k == 0:
                continue
            for i in grp:
                pb[i] = k
                members.append(i)
            offs.append(len(members))
        return pb, np.array(offs, np.int32), np.array(members, np.int32)

    def refcount(self, block: int) -> int:
        return self.ref[block]

    def stats(self):
        """(free, used, shared, utilisation); utilisation = filled slots of the
        used blocks / (16 * used blocks)."""
        free = len(self.free)
        used = self.num_blocks - free
        shared = sum(1 for r in self.ref if r > 1)
        fill = {}
        for s, blocks in self.tables.items():
            if s in self.swapped:
                continue
            n = self.lens[s]
            for j, b in enumerate(blocks):
                fill[b] = max(fill.get(b, 0), min(BLOCK_TOKENS, n - j * BLOCK_TOKENS))
        util = (sum(fill.values()) / (BLOCK_TOKENS * used)) if used else 0.0
        return free, used, shared, util
