"""Reference model of the host block manager (test infrastructure; only tests/ use it).

The pages fix the idea, not a policy:
 * "vLLM — PagedAttention으로 LLM 추론 성능을 2~4배 끌어올린 서빙 엔진" (dev.to),
   section "PagedAttention — OS 가상 메모리에서 영감": blocks are handed out
   only as tokens arrive, free blocks serve any other request, and logical
   blocks map to physical blocks through a per-sequence table.
 * "Nano-vLLM로 배우는 vLLM 추론 엔진 작동 원리 한눈에 정리" (tilnote.io),
   section "KV 캐시와 Block Manager": the block manager keeps block metadata on
   the CPU while the K/V tensors stay on the GPU; prefix blocks can be shared.

The policy modelled here (the library implements the same one, separately):
 * the free blocks form a stack; ``free_order[0]`` is handed out first;
 * a block's reference count is the number of tables that hold it; a block
   returns to the top of the stack when its count reaches zero;
 * releasing a sequence walks its table from logical block 0 upwards;
 * appending a token at position p allocates a block when p % Bs == 0 and
   the token's slot is table[p // Bs] * Bs + p % Bs;
 * a batch append is all-or-nothing: if the free stack cannot cover every new
   block it needs, nothing changes;
 * append_tokens refuses to append into a block that another table also holds
   (append_token_ids copies it instead, below).

Prefix caching and copy-on-write (the model of pa_bm_add_seq_tokens,
pa_bm_append_token_ids and pa_bm_fork_all):
 * Nano-vLLM page, section "KV 캐시와 Block Manager": requests that share the
   front of a prompt share its blocks, which are identified by a hash and
   reused without recomputation.  Reading: a FULL block is identified by the
   64-bit FNV-1a hash of (its parent's hash as 8 little-endian bytes, then its
   Bs token ids as 4 little-endian bytes each); the first block's parent hash
   is 0.  A lookup hits only if the stored token ids are equal too.
 * vLLM overview page, section "PagedAttention — OS 가상 메모리에서 영감": the
   pool is paged like OS virtual memory.  Reading: as in OS paging, a write
   into a page that several tables share copies it first (copy-on-write): the
   writer gets a fresh block, the copy (src, dst) is reported for the device,
   and the old block loses one reference.
 * The free list keeps blocks in order; allocation takes the top.  A block
   released without a hash goes on top (so without hashes this is exactly
   the stack above); a block released with a hash goes to the bottom, and a
   sequence's cached blocks go there tail first, so the oldest cached blocks
   are evicted first and a prefix root after its descendants.  Taking a
   cached block from the list evicts its hash; a hit on a cached free block
   takes it out of the list.
 * A sequence's blocks are hashed only while every token has an id
   (admitted with pa_bm_add_seq_tokens, grown with pa_bm_append_token_ids, or
   forked whole from such a sequence); a block is registered when it fills,
   unless its hash is already registered.
"""
from __future__ import annotations

FNV_OFFSET = 0xCBF29CE484222325
FNV_PRIME = 0x100000001B3
MASK64 = (1 << 64) - 1


def fnv1a64(data: bytes, h: int = FNV_OFFSET) -> int:
    """64-bit FNV-1a: for each byte, h ^= byte, then h *= prime (mod 2^64)."""
    for byte in data:
        h ^= byte
        h = (h * FNV_PRIME) & MASK64
    return h


def block_hash(parent: int, token_ids) -> int:
    data = int(parent).to_bytes(8, "little") + b"".join(int(t).to_bytes(4, "little", signed=True)
                                                        for t in token_ids)
    return fnv1a64(data)


class OutOfBlocks(RuntimeError):
    pass


class SharedBlockWrite(RuntimeError):
    pass


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int, max_seqs: int, max_blocks_per_seq: int,
                 free_order):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.max_seqs = max_seqs
        self.max_blocks_per_seq = max_blocks_per_seq
        self.free = [int(b) for b in reversed(list(free_order))]  # top = end of the list
        self.ref = [0] * num_blocks
        self.tables = [[] for _ in range(max_seqs)]
        self.lens = [0] * max_seqs
        self.live = [False] * max_seqs
        # prefix caching
        self.cache = {}                          # hash -> block
        self.bhash = [None] * num_blocks         # registered hash of a block
        self.ids = [None] * num_blocks           # token ids held by a block ([Bs], None = unknown)
        self.chain = [0] * max_seqs              # hash of a sequence's last full block
        self.hashable = [False] * max_seqs       # every token of the sequence has an id

    # -- pool ---------------------------------------------------------------
    def _pop(self) -> int:
        blk = self.free.pop()
        if self.bhash[blk] is not None:          # evict
            del self.cache[self.bhash[blk]]
            self.bhash[blk] = None
        self.ref[blk] = 1
        self.ids[blk] = [None] * self.block_size
        return blk

    def _release(self, blk: int) -> bool:
        """Drops one reference; True if the block became free (the caller files it)."""
        self.ref[blk] -= 1
        return self.ref[blk] == 0

    def _release_blocks(self, blocks) -> None:
        freed = [b for b in blocks if self._release(b)]
        for b in freed:                          # uncached: on top, in table order
            if self.bhash[b] is None:
                self.free.append(b)
        for b in reversed(freed):                # cached: to the bottom, tail first
            if self.bhash[b] is not None:
                self.free.insert(0, b)

    def _register(self, blk: int, h: int) -> None:
        if h not in self.cache and self.bhash[blk] is None:
            self.cache[h] = blk
            self.bhash[blk] = h

    def num_free(self) -> int:
        return len(self.free)

    def num_cached(self) -> int:
        return len(self.cache)

    # -- sequences ----------------------------------------------------------
    def import_seq(self, seq: int, length: int, blocks) -> None:
        """Adopt a sequence whose blocks were laid out outside the free stack."""
        assert not self.live[seq]
        blocks = [int(b) for b in blocks]
        assert len(blocks) == -(-length // self.block_size)
        for blk in blocks:
            self.ref[blk] += 1
        self.tables[seq] = blocks
        self.lens[seq] = length
        self.live[seq] = True
        self.hashable[seq] = False

    def add_seq(self, seq: int, length: int) -> None:
        """Admit a sequence of `length` cached tokens into fresh blocks."""
        assert not self.live[seq]
        need = -(-length // self.block_size)
        if need > len(self.free):
            raise OutOfBlocks(seq)
        self.tables[seq] = [self._pop() for _ in range(need)]
        self.lens[seq] = length
        self.live[seq] = True
        self.hashable[seq] = False

    def free_seq(self, seq: int) -> None:
        assert self.live[seq]
        self._release_blocks(self.tables[seq])
        self.tables[seq] = []
        self.lens[seq] = 0
        self.live[seq] = False
        self.hashable[seq] = False
        self.chain[seq] = 0

    def append_tokens(self, seqs) -> list:
        """One new token for each listed sequence; returns the slots."""
        Bs = self.block_size
        need = 0
        for seq in seqs:
            p = self.lens[seq]
            if p % Bs == 0:
                need += 1
            elif self.ref[self.tables[seq][p // Bs]] > 1:
                raise SharedBlockWrite(seq)
        if need > len(self.free):
            raise OutOfBlocks(need)
        slots = []
        for seq in seqs:
            p = self.lens[seq]
            if p % Bs == 0:
                self.tables[seq].append(self._pop())
            slots.append(self.tables[seq][p // Bs] * Bs + p % Bs)
            self.lens[seq] = p + 1
            self.hashable[seq] = False
        return slots

    # -- prefix caching and copy-on-write --------------------------------------
    def add_seq_tokens(self, seq: int, token_ids) -> int:
        """Admit a sequence by its token ids, reusing the cached blocks of its longest cached
        prefix of full blocks; returns the number of tokens found cached."""
        assert not self.live[seq]
        Bs = self.block_size
        ids = [int(t) for t in token_ids]
        n = len(ids)
        full, nb = n // Bs, -(-n // Bs)
        hits, parent = [], 0
        for i in range(full):
            chunk = ids[i * Bs:(i + 1) * Bs]
            h = block_hash(parent, chunk)
            b = self.cache.get(h)
            if b is None or self.ids[b] != chunk:
                break
            hits.append(b)
            parent = h
        free_hits = sum(1 for b in hits if self.ref[b] == 0)
        if nb - len(hits) > len(self.free) - free_hits:
            raise OutOfBlocks(seq)
        for b in hits:
            if self.ref[b] == 0:
                self.free.remove(b)
            self.ref[b] += 1
        blocks = list(hits)
        for i in range(len(hits), nb):
            b = self._pop()
            chunk = ids[i * Bs:(i + 1) * Bs]
            self.ids[b] = chunk + [None] * (Bs - len(chunk))
            if i < full:
                h = block_hash(parent, chunk)
                self._register(b, h)
                parent = h
            blocks.append(b)
        self.tables[seq] = blocks
        self.lens[seq] = n
        self.live[seq] = True
        self.hashable[seq] = True
        self.chain[seq] = parent
        return len(hits) * Bs

    def fork_all(self, seq: int, src: int) -> None:
        """Admit seq sharing every block of src, its partial last block included."""
        assert not self.live[seq] and self.live[src] and seq != src
        for b in self.tables[src]:
            self.ref[b] += 1
        self.tables[seq] = list(self.tables[src])
        self.lens[seq] = self.lens[src]
        self.live[seq] = True
        self.hashable[seq] = self.hashable[src]
        self.chain[seq] = self.chain[src]

    def append_token_ids(self, seqs, token_ids):
        """One new token (with its id) per listed sequence.  A token whose block is shared
        gets a private copy first.  Returns (slots, copies [(src, dst)])."""
        Bs = self.block_size
        need = 0
        for seq in seqs:
            p = self.lens[seq]
            if p % Bs == 0 or self.ref[self.tables[seq][p // Bs]] > 1:
                need += 1
        if need > len(self.free):
            raise OutOfBlocks(need)
        slots, copies = [], []
        for seq, tid in zip(seqs, token_ids):
            p = self.lens[seq]
            t = self.tables[seq]
            if p % Bs == 0:
                t.append(self._pop())
            elif self.ref[t[p // Bs]] > 1:
                old = t[p // Bs]
                new = self._pop()
                self.ids[new] = list(self.ids[old])
                copies.append((old, new))
                t[p // Bs] = new
                self._release_blocks([old])
            b = t[p // Bs]
            self.ids[b][p % Bs] = int(tid)
            slots.append(b * Bs + p % Bs)
            self.lens[seq] = p + 1
            if (p + 1) % Bs == 0 and self.hashable[seq]:
                h = block_hash(self.chain[seq], self.ids[b])
                self._register(b, h)
                self.chain[seq] = h
        return slots, copies

    def table_array(self, seq: int):
        row = list(self.tables[seq])
        return row + [-1] * (self.max_blocks_per_seq - len(row))


class BlockPoolModel:
    """Model of the per-block pool (pa_pool_*): a stack of free ids and a count of holders.

    The pages give the idea (blocks handed out one at a time as tokens need them; a block of a
    shared prefix sits in several tables); the policy is the one the block manager above
    follows: free_order[0] is on top of the stack and handed out first, alloc of n is all or
    nothing, share adds a holder to an allocated block, free drops one and a block whose count
    reaches zero goes back on top.  Blocks not in free_order start allocated once.
    """

    def __init__(self, num_blocks: int, free_order=None):
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        assert len(set(order)) == len(order) and all(0 <= b < num_blocks for b in order)
        self.num_blocks = num_blocks
        self.refcount = [1] * num_blocks
        for b in order:
            self.refcount[b] = 0
        self.stack = list(reversed(order))          # top = end of the list

    def alloc(self, n: int):
        if n > len(self.stack):
            raise OutOfBlocks(n)
        out = []
        for _ in range(n):
            b = self.stack.pop()
            self.refcount[b] = 1
            out.append(b)
        return out

    def share(self, block: int) -> None:
        if not (0 <= block < self.num_blocks) or self.refcount[block] == 0:
            raise ValueError("share of a free or unknown block")
        self.refcount[block] += 1

    def free(self, block: int) -> None:
        if not (0 <= block < self.num_blocks) or self.refcount[block] == 0:
            raise ValueError("free of a free or unknown block")
        self.refcount[block] -= 1
        if self.refcount[block] == 0:
            self.stack.append(block)

    def num_free(self) -> int:
        return len(self.stack)
