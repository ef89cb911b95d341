"""Multi-scale retention on B200: thin Python binding over libretention.so."""
