"""Oracle model of the KV-cache block manager -- TEST INFRASTRUCTURE ONLY.

A plain Python restatement of the block-manager rules on the pages, used to check the native
allocator bit for bit (block ids, ref counts, slots, copy pairs).  It shares no code with it.

Rules followed (page title, section):
  * "PagedAttention原理", "从虚拟内存的启发": space is requested one block of B tokens at a time,
    only when the previous block is used up, so a sequence wastes fewer than B slots.
  * "PagedAttention原理", "实现一个虚拟内存" (block-table figure): each sequence maps logical block j
    to a physical block and records how many slots are filled.
  * "PagedAttention原理", "解决共享prompt" / "解决COW": every physical block has a reference count;
    a block shared by several logical blocks has count > 1 and is released only at 0.  Writing
    into a block with count 1 happens in place; otherwise: (1) allocate a new block, (2) copy the
    shared block into it, (3) map the sequence's logical block to the new block, (4) decrement the
    old block's count, (5) write the new data into the new block.
  * "PagedAttention原理", "COW 区别": a block with free slots is appended to, not copied.
  * "Paged Attention&Orca Paper笔记与解读", parallel sampling and beam search: sequences fork by
    sharing blocks; a block whose count drops to 0 is freed.

Readings where the pages are open:
  * The last block full: the next token gets a fresh block with no copy, even if the full block is
    shared.  Partial and shared: copy-on-write.  Partial and count 1: in place.
  * Free-block policy: a LIFO stack that starts as [n-1, ..., 1, 0], so the first allocation
    returns block 0 and a freed block is the next one handed out.
  * Freeing a sequence releases its blocks in logical order (j = 0, 1, ...).
  * Sequence ids are handed out 0, 1, 2, ... and never reused.
  * A reservation that cannot get every block it needs fails and changes nothing.
"""
from __future__ import annotations


class NoFreeBlock(RuntimeError):
    pass


class InvalidArg(ValueError):
    pass


class BlockManagerModel:
    def __init__(self, n_blocks: int, block_size: int):
        if n_blocks <= 0 or block_size <= 0:
            raise InvalidArg("n_blocks and block_size must be positive")
        self.n_blocks = n_blocks
        self.B = block_size
        self.ref = [0] * n_blocks
        self.free = list(range(n_blocks - 1, -1, -1))  # pop() -> 0 first
        self.seqs: dict[int, dict] = {}
        self._next_seq = 0

    # ---- blocks ---------------------------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free)

    def alloc_block(self) -> int:
        if not self.free:
            raise NoFreeBlock("pool exhausted")
        b = self.free.pop()
        self.ref[b] = 1
        return b

    def _check_block(self, b: int):
        if not (0 <= b < self.n_blocks) or self.ref[b] == 0:
            raise InvalidArg(f"block {b} is not allocated")

    def incref(self, b: int):
        self._check_block(b)
        self.ref[b] += 1

    def decref(self, b: int):
        self._check_block(b)
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    def refcount(self, b: int) -> int:
        if not (0 <= b < self.n_blocks):
            raise InvalidArg("block id out of range")
        return self.ref[b]

    # ---- sequences --------------------------------------------------------------------------
    def seq_create(self) -> int:
        sid = self._next_seq
        self._next_seq += 1
        self.seqs[sid] = {"table": [], "n": 0}
        return sid

    def _seq(self, sid: int) -> dict:
        if sid not in self.seqs:
            raise InvalidArg(f"unknown sequence {sid}")
        return self.seqs[sid]

    def seq_fork(self, parent: int) -> int:
        p = self._seq(parent)
        child = self.seq_create()
        for b in p["table"]:
            self.ref[b] += 1
        self.seqs[child] = {"table": list(p["table"]), "n": p["n"]}
        return child

    def seq_free(self, sid: int):
        s = self._seq(sid)
        for b in s["table"]:
            self.decref(b)
        del self.seqs[sid]

    def seq_len(self, sid: int) -> int:
        return self._seq(sid)["n"]

    def seq_table(self, sid: int) -> list[int]:
        return list(self._seq(sid)["table"])

    def reserve_slots(self, sid: int, n_new: int):
        """Reserve the next n_new token slots of a sequence.

        Returns (slots, cow_pairs): slot = physical_block * B + offset for each new token, and the
        (src, dst) block pairs whose contents must be copied before the new tokens are written.
        """
        s = self._seq(sid)
        if n_new < 0:
            raise InvalidArg("n_new must be >= 0")
        B, n, table = self.B, s["n"], s["table"]
        cow = 1 if (n_new > 0 and n % B != 0 and self.ref[table[-1]] > 1) else 0
        fresh = -(-(n + n_new) // B) - len(table)
        if cow + fresh > len(self.free):
            raise NoFreeBlock("pool exhausted")
        slots, pairs = [], []
        for _ in range(n_new):
            if n % B == 0:
                table.append(self.alloc_block())          # last block full (or none): fresh block
            elif self.ref[table[-1]] > 1:
                old = table[-1]                           # partial and shared: copy-on-write
                new = self.alloc_block()                  # (1) allocate
                pairs.append((old, new))                  # (2) copy old -> new (done by the caller)
                table[-1] = new                           # (3) remap the logical block
                self.decref(old)                          # (4) decrement the old count
            slots.append(table[n // B] * B + n % B)       # (5) the new token lands in the new block
            n += 1
        s["n"] = n
        return slots, pairs

    def build_block_tables(self, seq_ids, max_blocks_per_seq: int):
        """Pack the tables of seq_ids into [S][max_blocks_per_seq] (padding -1) plus the lengths."""
        tables, lens = [], []
        for sid in seq_ids:
            s = self._seq(sid)
            if len(s["table"]) > max_blocks_per_seq:
                raise InvalidArg("max_blocks_per_seq too small")
            tables.append(s["table"] + [-1] * (max_blocks_per_seq - len(s["table"])))
            lens.append(s["n"])
        return tables, lens
