"""libpaged: paged KV-cache decode attention for B200 (sm_100a), Python binding.

Placeholder until the binding lands.
"""
